// Device helpers of the mHC boundary kernels (sm_100a): PTX wrappers for the
// bulk-copy engine and mbarriers, bf16 packing, bounded waits, and the
// E8M0/E4M3 encoders of the MXFP8 layer input.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mhc.h"

namespace mhc {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- waits

// The bounded waits count SM cycles (clock64 is a register read; %globaltimer
// costs about a microsecond per read on this part). A budget of T ns is granted
// as 2*T cycles: at clocks up to 2 GHz the wait lasts at least T ns.
__device__ __forceinline__ long long wait_deadline(int64_t budget_ns) { return clock64() + 2 * budget_ns; }

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void record_error(unsigned* status, unsigned code) {
  if (status != nullptr) atomicCAS(status, 0u, code);
}

// ---------------------------------------------------------------- shared memory / TMA bulk copies

__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
  // make the initialised barrier visible to the async proxy (the TMA engine)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

// Wait for phase `parity` of `bar`, giving up at `deadline` (clock64 cycles).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, long long deadline) {
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() > deadline) return false;
  }
  return true;
}

// A 3-D box of a tensor map (this GPU's memory) into shared memory at dst, the
// transfer counted on `bar`; coordinates innermost first, x 16-byte aligned.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---------------------------------------------------------------- small async copies / L2 prefetch

// 4-byte global -> shared copy that does not occupy a register (LDGSTS); all
// copies of a thread complete at cp_async_wait_all.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most one (the most recent) committed group of this thread is in flight.
__device__ __forceinline__ void cp_async_wait_group1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// ---------------------------------------------------------------- global vector loads / stores

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {  // read-only, streaming
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 8-byte forms (4 bf16): the streaming kernel's lanes own 4 columns.
__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_cg_v2(const void* p) {  // L2 only: data other agents write
  uint2 v;
  asm volatile("ld.global.cg.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
// Maximum over the warp in one instruction (sm_100a); NaN inputs are skipped, as by fmaxf.
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint2 ld_volatile_v2(const void* p) {  // re-read on every call
  uint2 v;
  asm volatile("ld.volatile.global.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p) : "memory");
  return v;
}
// bf16 negative zero in both halves: the mark of a mailbox slot element that its
// producer has not written yet (a producer never stores negative zero).
constexpr unsigned kNegZero2 = 0x80008000u;
__device__ __forceinline__ bool has_neg_zero(const uint2 v) {
  return (__vcmpeq2(v.x, kNegZero2) | __vcmpeq2(v.y, kNegZero2)) != 0u;
}
// Negative zero halves of a bf16 pair replaced by positive zero.
__device__ __forceinline__ unsigned clear_neg_zero2(unsigned w) { return w & __vcmpne2(w, kNegZero2); }
__device__ __forceinline__ void st_v2(void* p, uint2 v) {
  asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
// 4 bf16 as two column pairs: f[m] = (element 2m, element 2m + 1).
__device__ __forceinline__ void unpack4x2(const uint2 v, float2 (&f)[2]) {
  f[0] = make_float2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u));
  f[1] = make_float2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
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

// ---------------------------------------------------------------- mailbox slots

// Producer side: one row of H bf16 (H a multiple of 8) into its slot with
// 16-byte stores, negative zeros made positive; thread t of nt takes every
// nt-th 8-element chunk. No fence and no flag follow: each element is its own
// "written" mark.
__device__ __forceinline__ void mailbox_store_row(__nv_bfloat16* slot, const __nv_bfloat16* src, int H, int t,
                                                  int nt) {
  for (int k = t * 8; k < H; k += nt * 8) {
    uint4 v = ld_nc_v4(src + k);
    v.x = clear_neg_zero2(v.x);
    v.y = clear_neg_zero2(v.y);
    v.z = clear_neg_zero2(v.z);
    v.w = clear_neg_zero2(v.w);
    st_v4(slot + k, v);
  }
}

// Consumer side: a slot's 4 elements as loaded, re-read until none is negative
// zero (bounded: on timeout the status records it and the values are used as
// they are).
__device__ __forceinline__ uint2 settle_slot(const __nv_bfloat16* src, uint2 v, long long deadline,
                                             unsigned* status) {
  while (has_neg_zero(v)) {
    if (clock64() > deadline) {
      record_error(status, MHC_ERR_DEVICE_TIMEOUT);
      break;
    }
    v = ld_volatile_v2(src);
  }
  return v;
}

// ---------------------------------------------------------------- warp-level tensor core MMA

// Four 8x8 b16 matrices from shared memory; lane l gives the row address of
// matrix l/8, row l%8 (the A operand of an m16n8k16 MMA).
__device__ __forceinline__ void ldmatrix_x4(unsigned (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}

// Two 8x8 b16 matrices (lanes 0-15 give the row addresses): the B operand.
__device__ __forceinline__ void ldmatrix_x2(unsigned (&r)[2], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(row_addr)));
}

// D = A * B + D, A 16x16 bf16 (row), B 16x8 bf16 (col), D 16x8 fp32.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const unsigned (&a)[4], const unsigned (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
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

// Approximate reciprocal (MUFU, <= 1 ulp): the Sinkhorn normalisations.
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
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

// ---------------------------------------------------------------- cross-block flags, dependent launch

__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// System scope: words that other GPUs write (peer stores over NVLink) or read.
__device__ __forceinline__ unsigned ld_acquire_sys(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_sys(unsigned* p, unsigned v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Programmatic dependent launch: wait for the preceding grid on the stream to
// complete (and its memory to be visible); a no-op when launched normally.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next grid on the stream (launched with programmatic serialization)
// to start once every block of this grid has executed this.
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace mhc
