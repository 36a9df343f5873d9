// Device helpers of the mHC boundary kernels (sm_100a): PTX wrappers for the
// bulk-copy engine and mbarriers, bf16 packing, bounded waits, and the
// E8M0/E4M3 encoders of the MXFP8 layer input.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mhc {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- timers / waits

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void record_error(unsigned* status, unsigned code) {
  atomicCAS(status, 0u, code);
}

// ---------------------------------------------------------------- shared memory / TMA bulk copies

__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// 1-D bulk copy global -> shared through the TMA engine; completion is counted
// in bytes on `bar`. dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar`, giving up at `deadline` (globaltimer ns).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, uint64_t deadline) {
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() > deadline) return false;
  }
  return true;
}

// ---------------------------------------------------------------- global vector loads / stores

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {  // read-only, streaming
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_v4(const void* p) {  // coherent (may alias an output)
  uint4 v;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------- bf16 packing

// 8 bf16 in a uint4: element 2m in the low half of word m, 2m+1 in the high half.
__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
  const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    f[2 * m] = __uint_as_float(w[m] << 16);
    f[2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
  }
}

__device__ __forceinline__ unsigned pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<unsigned*>(&b);
}

// Round 8 floats to bf16 (RNE), return packed and the rounded values as floats.
__device__ __forceinline__ uint4 round8(const float (&f)[8], float (&r)[8]) {
  uint4 v;
  v.x = pack_bf16x2(f[0], f[1]);
  v.y = pack_bf16x2(f[2], f[3]);
  v.z = pack_bf16x2(f[4], f[5]);
  v.w = pack_bf16x2(f[6], f[7]);
  unpack8(v, r);
  return v;
}

// ---------------------------------------------------------------- MXFP8 encoders

// Exponent e of an MXFP8 block whose largest magnitude is `amax` (a finite,
// non-negative float): the smallest e with amax <= 448 * 2^e, clamped to
// [-127, 127]. With amax = m * 2^q, m in [1, 2): e = q - 8 if m <= 1.75
// (448 = 1.75 * 2^8) else q - 7. Read from the float's bits: no log, no division.
__device__ __forceinline__ int e8m0_exponent(float amax) {
  const unsigned u = __float_as_uint(amax);
  const int biased = static_cast<int>(u >> 23);
  if (biased == 0) return -127;  // zero or subnormal: below 2^-126, the clamp decides
  const int q = biased - 127;
  const unsigned frac = u & 0x7fffffu;
  int e = (frac <= 0x600000u) ? q - 8 : q - 7;  // 0x600000 is the fraction of 1.75
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as a float for e in [-127, 121] (the range finite bf16 blocks reach).
__device__ __forceinline__ float exp2_neg(int e) { return __uint_as_float(static_cast<unsigned>(127 - e) << 23); }

// Two floats to two E4M3 bytes (RNE, saturating to +-448): `lo` lands in the
// low byte of the result, `hi` in the high byte.
__device__ __forceinline__ unsigned short e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- grid barrier

// Self-resetting barrier over all blocks of the grid, with a bounded wait.
// ctl[kBarCount] counts arrivals, ctl[kBarGen] is the generation. A block reads
// the generation before it arrives; the last arriver resets the count and then
// bumps the generation, which releases the others. Every block must call it the
// same number of times. Returns false (and records MHC_ERR_DEVICE_TIMEOUT) when
// the wait ran past `deadline`; the barrier state is then unusable until the
// workspace is zeroed again.
__device__ __forceinline__ bool grid_barrier(unsigned* count, unsigned* gen, unsigned expected,
                                             unsigned* status, uint64_t deadline, unsigned timeout_code,
                                             int* flag_smem) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    const unsigned my_gen = ld_acquire_gpu(gen);
    const unsigned old = atomicAdd(count, 1u);
    if (old == expected - 1) {
      atomicExch(count, 0u);
      __threadfence();
      atomicAdd(gen, 1u);
    } else {
      while (ld_acquire_gpu(gen) == my_gen) {
        if (global_ns() > deadline) {
          record_error(status, timeout_code);
          ok = false;
          break;
        }
        __nanosleep(20);
      }
    }
    *flag_smem = ok ? 1 : 0;
  }
  __syncthreads();
  return *flag_smem != 0;
}

}  // namespace mhc
