// Concurrency check of the mailbox slot protocol (test infrastructure, not part
// of the library). The protocol is the one of the pages' BoundaryAllReduce
// (publish_target / mark_published on the producer side, the collecting
// __call__ on the consumer side): a slot element holding bf16 negative zero has
// not been written yet, a producer never stores negative zero, and the consumer
// re-reads an element until it is written, then puts the mark back.
//
// One cooperative launch plays a whole round: its first W blocks are the
// producers, each storing its R rows into the consumer's slots with the
// library's producer step (mailbox_store_row) after a per-row delay, while the
// other blocks are the consumer, reading the same slots as they fill with the
// library's bounded slot wait (settle_slot), summing them in producer order in
// fp32 and re-marking them. The cooperative launch makes every block resident
// at once, so the consumer's waits run while the stores are really in flight;
// every wait is bounded (the producers' delays by their cycle counts, the
// consumer's slot waits by its deadline).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mhc_device.cuh"

namespace {

using namespace mhc;

constexpr int kThreads = 256;
constexpr int kMaxProducers = 16;
constexpr int kMaxDelayCycles = 8000000;  // about 4 ms at the part's clocks

struct RaceParams {
  const __nv_bfloat16* x;   // [W][R][H] the producers' rows
  __nv_bfloat16* slots;     // [W][R][H] the consumer's slots of one parity
  float* sum;               // [R][H] the consumer's sums, producers added in order 0..W-1
  unsigned* status;         // [0] first error code, [1] 8-byte groups first loaded unwritten
  const int* delay_cycles;  // [W][R] producer w stores row r this many cycles after it starts; < 0: never
  int W, R, H, consumers;
  int64_t budget_ns;
};

__global__ void __launch_bounds__(kThreads) mailbox_race_kernel(const RaceParams p) {
  const int tid = threadIdx.x;
  if (static_cast<int>(blockIdx.x) < p.W) {  // producer w
    const int w = blockIdx.x;
    const long long t0 = clock64();
    for (int r = 0; r < p.R; ++r) {
      const int d = p.delay_cycles[w * p.R + r];
      if (d < 0) continue;
      while (clock64() - t0 < d) {
      }
      const size_t off = (static_cast<size_t>(w) * p.R + r) * p.H;
      mailbox_store_row(p.slots + off, p.x + off, p.H, tid, kThreads);
    }
    return;
  }
  // consumer block c takes 4-column groups c*256 + tid, c*256 + tid + consumers*256, ... of every row
  const int c = blockIdx.x - p.W;
  const long long deadline = wait_deadline(p.budget_ns);
  unsigned early = 0;
  for (int r = 0; r < p.R; ++r) {
    for (int k = (c * kThreads + tid) * 4; k < p.H; k += p.consumers * kThreads * 4) {
      float2 xs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      for (int u = 0; u < p.W; ++u) {
        const __nv_bfloat16* src = p.slots + (static_cast<size_t>(u) * p.R + r) * p.H + k;
        uint2 v = ld_cg_v2(src);
        if (has_neg_zero(v)) ++early;
        v = settle_slot(src, v, deadline, p.status);
        float2 f[2];
        unpack4x2(v, f);
        xs[0] = __fadd2_rn(xs[0], f[0]);
        xs[1] = __fadd2_rn(xs[1], f[1]);
      }
      for (int u = 0; u < p.W; ++u)
        st_v2(p.slots + (static_cast<size_t>(u) * p.R + r) * p.H + k, make_uint2(kNegZero2, kNegZero2));
      *reinterpret_cast<float4*>(p.sum + static_cast<size_t>(r) * p.H + k) =
          make_float4(xs[0].x, xs[0].y, xs[1].x, xs[1].y);
    }
  }
  if (early != 0u) atomicAdd(p.status + 1, early);
}

bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

}  // namespace

// Runs one round on `stream` (a cudaStream_t, or null). x [W][R][H] bf16, slots
// [W][R][H] bf16 (negative zero where unwritten, as mhc_mailbox_init leaves
// them), sum [R][H] fp32, status 2 words zeroed by the caller, delay_cycles
// [W][R] int32, all device memory, 16-byte aligned. 1 <= W <= 16, R >= 1, H a
// positive multiple of 8, consumers >= 1, 0 <= delays <= 8e6 or negative.
// Returns 0, -1 for an argument outside these bounds (nothing launched), or
// the CUDA error of the launch.
extern "C" __attribute__((visibility("default"))) int mhc_race_run(const void* x, void* slots, float* sum,
                                                                    unsigned* status, const int* delay_cycles,
                                                                    int W, int R, int H, int consumers,
                                                                    int64_t budget_ns, void* stream) {
  if (!x || !slots || !sum || !status || !delay_cycles) return -1;
  if (!aligned16(x) || !aligned16(slots) || !aligned16(sum)) return -1;
  if (W < 1 || W > kMaxProducers || R < 1 || H < 8 || H % 8 != 0 || consumers < 1 || consumers > 128) return -1;
  if (budget_ns < 0 || budget_ns > 10000000000LL) return -1;
  RaceParams p{static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(slots), sum, status,
               delay_cycles, W, R, H, consumers, budget_ns};
  void* args[] = {&p};
  const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(mailbox_race_kernel),
                                                    dim3(W + consumers), dim3(kThreads), args, 0,
                                                    static_cast<cudaStream_t>(stream));
  return static_cast<int>(e);
}

extern "C" __attribute__((visibility("default"))) int mhc_race_max_delay_cycles() { return kMaxDelayCycles; }
