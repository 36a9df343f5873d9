// mHC decode boundary on B200 (sm_100a): the fused kernel and the C ABI of
// libmhc.so (declared in include/mhc.h).
//
// A boundary is two launches chained by programmatic dependent launch (PDL).
// The streaming kernel (boundary_kernel): block g owns columns [64g, 64g+64)
// of H for every row, so each weight of fn is read from HBM exactly once.
//   1. A TMA bulk copy brings the block's fn slice into shared memory (packed
//      bf16 terms, or fp32 that the block splits into bf16 terms while its row
//      data are in flight) and the block's activations are prefetched into L2,
//      both before the kernel waits for its predecessor on the stream;
//   2. per (row, 4 columns) a lane sums the partials (local buffers, peers'
//      buffers, or the slots of a publish/collect mailbox as they fill; up to
//      16 rows of local partials arrive by two tensor-map copies) or
//      finalizes the MoE output, applies the mHC post-mix (vllm
//      ...boundary.boundary, Boundaries.post_only: mhc_post(x, residual, post,
//      comb)), rounds the new streams to bf16, stores them, sums the squares of
//      their collapse with the carried pre (BoundaryState.pre) and of the streams;
//   3. the block projects its rows' n*64 stream values onto the C fn columns on
//      the tensor cores (mma.sync bf16, fn as three bf16 terms; single or paired
//      16-row tiles per warp by row count) and writes its partial sums to the
//      workspace.
// The tail kernel (boundary_tail_kernel), once the streaming kernel is done:
//   4. layer-input blocks normalise 256-column tasks of the rows into the layer
//      input (and MXFP8); beside them, coefficient blocks (placed first for 4-32
//      rows, so that they start on the SMs the streaming kernel leaves free)
//      finish the rows' coefficients (logits, sigmoid, Sinkhorn on scale vectors
//      in one thread per row).
// The residual-only variant is the streaming kernel alone. All reductions run
// in a fixed order, so results are bitwise reproducible.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <cstring>
#include <map>
#include <mutex>

#include "../../include/mhc.h"
#include "mhc_device.cuh"

namespace mhc {

constexpr int kCols = 64;      // columns of H per block
constexpr int kThreads = 256;  // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRows = 128;
constexpr int kMaxPartials = 16;
constexpr int kMaxTopK = 16;
constexpr int kMaxIters = 1000;
constexpr int kMaxBlocks = 148;  // most H/64 blocks: the tail's per-lane loads are sized for it
constexpr int kPrefetchRows = 64;  // the streaming kernel prefetches its rows into L2 up to this many
constexpr int kPrefetchPartRows = 96;  // and its first kPrefetchRows rows up to this many
// Workspace header: the status word (byte 0); the partial sums follow.
constexpr size_t kWsHeader = 1024;
constexpr int kStatusWord = 0;

enum Front { kPartials = 0, kMoe = 1, kStreams = 2, kBroadcast = 3, kMailbox = 4 };
// Fronts whose x is a sum of P bf16 partials (kMailbox: slots of a mailbox that
// producers fill concurrently, each element valid once it is not negative zero).
__host__ __device__ constexpr bool sums_partials(int front) { return front == kPartials || front == kMailbox; }

__host__ __device__ constexpr int logits_of(int n) { return 2 * n + n * n; }
// logit count padded to a multiple of 4 (the tail's base array in shared memory)
__host__ __device__ constexpr int cpad_of(int n) { return (logits_of(n) + 3) & ~3; }
// Per-block record of a row in the workspace: C dot products, then sum v^2,
// padded to a power of two >= 8 floats.
__host__ __device__ constexpr int red_of(int n) {
  return logits_of(n) + 1 <= 8 ? 8 : (logits_of(n) + 1 <= 16 ? 16 : 32);
}
// fp32 fn slice in shared memory as the bulk copies land it (unpacked fn): pieces
// of 8 rows of C floats followed by a 16-byte gap, which spreads the split
// loop's reads over the banks.
__host__ __device__ constexpr int fn_piece_bytes(int n) { return 8 * logits_of(n) * 4 + 16; }

struct Params {
  // front ends
  const __nv_bfloat16* pptr[kMaxPartials];  // partial u: [R, H] at pptr[u]
  int premote;  // partials may be other GPUs' memory: L2-only loads, no prefetch
  int P;
  const __nv_bfloat16* gemm2;
  int num_perm;
  const float* ew;
  const int32_t* e2p;
  int topk;
  const __nv_bfloat16* shared_out;
  const __nv_bfloat16* residual;
  const __nv_bfloat16* x;
  const float* post;
  const float* comb;
  const float* pre;  // carried pre (boundary) or pre_mix (coefficients entry)
  // tail
  const __nv_bfloat16* norm_weight;
  float norm_eps;
  const float* fn;
  const __nv_bfloat16* fn_packed;  // [G][3][CP8][n*64 + 8] bf16 terms of fn, or null
  const float* scale;
  const float* base;
  float rms_eps, pre_eps, sk_eps, alpha;
  int iters;
  __nv_bfloat16* residual_out;
  __nv_bfloat16* aux_out;  // stream mean of the new streams [R, H], or null
  __nv_bfloat16* layer_input;
  uint8_t* q_data;
  uint8_t* q_scale;
  int q_swizzled;
  float* post_out;
  float* comb_out;
  float* pre_out;
  int R, H;
  int write_res, do_layer, do_coeff;
  // workspace
  unsigned* ctl;
  float* sc2_part;  // [R][G]
  float* dot_part;  // [R][G][RED]
  // the streams the tail normalises: the new streams, the given streams, or the
  // embedding of the first layer (whose identity pre-mix selects it)
  const __nv_bfloat16* tail_streams;
  int tail_broadcast;
  int tail_layer_blocks;  // tail blocks that write the layer input (or 0)
  int tail_coeff_blocks;  // tail blocks that finish the coefficients of rows j, j + this, ...
  int tail_coeff_first;   // coefficient blocks take the tail's first block indices
  int extra_tx;  // test hook: 16-byte units the fn wait expects beyond what arrives
  int64_t budget_ns;
  int staged;  // the partials and streams arrive by tensor-map copies (kPartials, rows <= kStagedRows)
};

// Up to this many rows, the partials front brings a block's partials and streams
// into shared memory with two tensor-map copies instead of per-lane loads
// (B200, us per boundary, staged / per-lane: 6.57 / 6.70-6.75 at 16 rows, equal
// within 0.03 at 1 and 8 rows, 7.69-7.89 / 7.66-7.72 at 32 rows).
constexpr int kStagedRows = 16;

struct SmemLayout {
  int fn_off, bs_off, v_off, mix_off, moe_off, st_off, misc_off, total;
};

// Projection operands: n-tiles of 8 logit columns; staged stream rows and fn
// columns are n*64 bf16 plus a 16-byte gap (ldmatrix rows in distinct banks).
__host__ __device__ constexpr int ntiles_of(int n) { return (logits_of(n) + 7) / 8; }
__host__ __device__ constexpr int kstride_of(int n) { return n * kCols + 8; }

// Shared memory of the streaming kernel (packed: fn arrives already split, so
// the fp32 staging area is not needed).
template <int N>
__host__ __device__ inline SmemLayout smem_layout(int R, int topk, bool moe, bool packed, int staged_p = 0) {
  constexpr int CP8 = ntiles_of(N) * 8;
  SmemLayout L{};
  int o = 0;
  L.fn_off = o;  // fn slice as the bulk copies land it
  if (!packed) o += N * 8 * fn_piece_bytes(N);
  L.bs_off = o;  // fn slice as three bf16 terms, [3][CP8][n*64 + 8]
  o += 3 * CP8 * kstride_of(N) * 2;
  L.v_off = o;  // new streams, bf16 [roundup(R, 16)][n*64 + 8]
  o += ((R + 15) & ~15) * kstride_of(N) * 2;
  L.mix_off = o;  // [R][post n | comb n*n | pre n]
  o += R * (2 * N + N * N) * 4;
  o = (o + 15) & ~15;
  L.moe_off = o;
  if (moe) o += R * topk * 8;
  o = (o + 127) & ~127;
  L.st_off = o;  // staged rows: partials [P][R][64 cols], then streams [R][n][64 cols], bf16
  o += staged_p > 0 ? (staged_p + N) * R * kCols * 2 : 0;
  L.misc_off = o;  // mbarriers: fn slice, staged rows
  o += 16;
  L.total = o;
  return L;
}

// Shared memory of the tail kernel.
struct TailLayout {
  int part_off, cst_off, total;
};

template <int N>
__host__ __device__ inline TailLayout tail_layout() {
  constexpr int CP = cpad_of(N);
  TailLayout L{};
  int o = 0;
  L.part_off = o;  // [kWarps rows][kWarps][RED] floats: the warps' shares of a row's records
  o += kWarps * kWarps * red_of(N) * 4;
  L.cst_off = o;  // scale[4], base[CP]
  o += (4 + CP) * 4;
  L.total = (o + 15) & ~15;
  return L;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

__device__ __forceinline__ float sum16_lanes(float v) {  // over the 16 lanes sharing lane bit 4
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

__device__ __forceinline__ int swizzled_scale_offset(int r, int c, int col_tiles) {
  const int tile = (r >> 7) * col_tiles + (c >> 2);
  const int rr = r & 127;
  return tile * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3);
}

// Registers of one row-pair step of a lane (4 columns of one row): the stream
// vectors and up to 8 partial (or gathered) vectors, plus the shared-output /
// embedding vector.
template <int N>
struct PairLoads {
  uint2 rv[N];
  uint2 pv[8];
  uint2 sv;
};
// The streaming kernel runs 16 warps; a warp covers a row pair x 64 columns,
// a lane 4 columns of one row.
constexpr int kT1 = 512;
constexpr int kW1 = kT1 / 32;

template <int N, int FRONT>
__device__ __forceinline__ void load_pair(const Params& p, int r, int h0, const int* e2p_s, PairLoads<N>& Q) {
  const int H = p.H;
  if (r >= p.R) return;
  if constexpr (FRONT == kBroadcast) {
    Q.sv = ld_nc_v2(p.x + static_cast<size_t>(r) * H + h0);
  } else {
#pragma unroll
    for (int j = 0; j < N; ++j) Q.rv[j] = ld_v2(p.residual + (static_cast<size_t>(r) * N + j) * H + h0);
  }
  if (sums_partials(FRONT)) {
    const size_t off = static_cast<size_t>(r) * H + h0;
    if (FRONT == kMailbox || p.premote) {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < p.P) Q.pv[u] = ld_cg_v2(p.pptr[u] + off);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < p.P) Q.pv[u] = ld_nc_v2(p.pptr[u] + off);
    }
  } else if (FRONT == kMoe) {
    Q.sv = ld_nc_v2(p.shared_out + static_cast<size_t>(r) * H + h0);
    const int* idx = e2p_s + r * p.topk;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (u < p.topk) {
        const int e = idx[u];
        Q.pv[u] = (e >= 0 && e < p.num_perm) ? ld_nc_v2(p.gemm2 + static_cast<size_t>(e) * H + h0)
                                             : make_uint2(0, 0);
      }
    }
  }
}

// fn as three bf16 terms, f = hi + mid + lo to 2^-24: each bf16 x bf16 product is
// exact in fp32, so three tensor-core products return the fp32 projection up to
// the order of the fp32 additions.
__device__ __forceinline__ void split3(float f, __nv_bfloat16& hi, __nv_bfloat16& mid, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(f);
  const float r1 = f - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r1);
  lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
}

// Bytes of a block's packed fn slice: the B operand of the projection exactly as
// it sits in shared memory, [3][CP8][n*64 + 8] bf16.
__host__ __device__ constexpr int packed_slice_bytes(int n) { return 3 * ntiles_of(n) * 8 * kstride_of(n) * 2; }
static_assert(packed_slice_bytes(1) % 16 == 0 && packed_slice_bytes(2) % 16 == 0 && packed_slice_bytes(4) % 16 == 0,
              "a bulk copy moves a multiple of 16 bytes");

// 80 registers a thread: 512 threads leave room on the SM for the tail kernel's
// blocks, which launch early (programmatic dependent launch).
// PAIRED: the projection takes pairs of row tiles (launched from four row tiles
// on; a separate instantiation, so that the other keeps its registers and code).
template <int N, int FRONT, bool PAIRED>
__global__ void __maxnreg__(80) boundary_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_part,
                                                const __grid_constant__ CUtensorMap tm_res) {
  constexpr int C = logits_of(N);
  constexpr int KC = N * kCols;       // stream values per row in this block
  constexpr int KS = kstride_of(N);   // staged row stride (bf16)
  constexpr int NT = ntiles_of(N);    // 8-column tiles of the projection
  constexpr int CP8 = NT * 8;
  constexpr int RED = red_of(N);
  constexpr int MIX = 2 * N + N * N;
  constexpr int PIECE = fn_piece_bytes(N);
  extern __shared__ __align__(128) unsigned char smem[];
  const bool staged = FRONT == kPartials && p.staged != 0;
  const SmemLayout L = smem_layout<N>(p.R, p.topk, FRONT == kMoe, p.fn_packed != nullptr, staged ? p.P : 0);
  unsigned char* fn_s = smem + L.fn_off;
  __nv_bfloat16* bs_s = reinterpret_cast<__nv_bfloat16*>(smem + L.bs_off);
  __nv_bfloat16* v_s = reinterpret_cast<__nv_bfloat16*>(smem + L.v_off);
  float* mix_s = reinterpret_cast<float*>(smem + L.mix_off);
  int* e2p_s = reinterpret_cast<int*>(smem + L.moe_off);
  float* ew_s = reinterpret_cast<float*>(smem + L.moe_off) + p.R * p.topk;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.misc_off);
  uint64_t* sbar = bar + 1;  // the staged rows
  const unsigned char* st_s = smem + L.st_off;

  const int g = blockIdx.x;
  const int G = gridDim.x;
  const int H = p.H;
  const int R = p.R;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rq = lane >> 4, vec = lane & 15;
  const int h0 = g * kCols + vec * 4;  // this lane's 4 columns in the row-pair phase
  const long long deadline = wait_deadline(p.budget_ns);
  unsigned* status = p.ctl + kStatusWord;
  const int npairs = (R + 1) >> 1;

  // ---- 1. the block's fn slice by TMA bulk copies. Weights are never written by
  // the kernel that precedes this one on the stream, so this runs before the
  // wait on that kernel (programmatic dependent launch).
  const bool packed = p.fn_packed != nullptr;
  if (staged && tid == 0) {
    mbar_init(sbar, 1);
    prefetch_tensormap(&tm_part);
    prefetch_tensormap(&tm_res);
  }
  if (p.do_coeff) {
    if (tid == 0) mbar_init(bar, 1);
    __syncthreads();
    if (packed) {  // pre-split terms (mhc_projection_pack): one copy, waited for at step 5
      if (tid == 0) {
        constexpr int PB = packed_slice_bytes(N);
        mbar_arrive_expect_tx(bar, PB + 16 * p.extra_tx);
        bulk_g2s(bs_s, reinterpret_cast<const unsigned char*>(p.fn_packed) + static_cast<size_t>(g) * PB, PB, bar);
      }
    } else if (warp == 0) {
      if (lane == 0) mbar_arrive_expect_tx(bar, KC * C * 4 + 16 * p.extra_tx);
      __syncwarp();
      for (int m = lane; m < N * 8; m += 32) {
        const int i = m >> 3, piece = m & 7;
        bulk_g2s(fn_s + m * PIECE, p.fn + (static_cast<size_t>(i) * H + g * kCols + piece * 8) * C, 8 * C * 4, bar);
      }
    }
  }

  // ---- 2. bring this block's activations into L2 while the preceding kernel may
  // still run: a prefetch is only a hint and L2 is the point of coherence, so
  // it is safe before the wait; gather indices read now only steer prefetches.
  // Every row up to 64 rows; the first 64 rows up to 96 (the paired
  // instantiation, which serves 49 rows and more, except the MoE gathers); past that the prefetches
  // cost more than they save (us per boundary with / without, B200: 7.65 / 8.23
  // at 32 rows, 9.81 / 10.20 at 48; all 96 rows 15.79 / 15.45, the first 64 of
  // 96 13.84 / 14.09; the first 64 of 128 16.27 / 16.02).
  constexpr bool kPart = PAIRED && FRONT != kMoe;  // (the gathers keep the 64-row limit)
  const int pf_rows = kPart ? (R <= kPrefetchRows ? R : (R <= kPrefetchPartRows ? kPrefetchRows : 0)) : R;
  if ((vec == 0 || vec == 15) && (kPart ? pf_rows > 0 : R <= kPrefetchRows)) {
    for (int q = warp; q < npairs; q += kW1) {
      const int r = q * 2 + rq;
      if (r >= pf_rows) break;
      if constexpr (FRONT == kBroadcast) {
        prefetch_l2(p.x + static_cast<size_t>(r) * H + h0);
      } else {
        for (int j = 0; j < N; ++j) prefetch_l2(p.residual + (static_cast<size_t>(r) * N + j) * H + h0);
      }
      if (sums_partials(FRONT)) {  // (a mailbox's slots are this GPU's memory)
        if (FRONT == kMailbox || !p.premote)
          for (int pp = 0; pp < p.P; ++pp) prefetch_l2(p.pptr[pp] + static_cast<size_t>(r) * H + h0);
      } else if (FRONT == kMoe) {
        prefetch_l2(p.shared_out + static_cast<size_t>(r) * H + h0);
        for (int t = 0; t < p.topk; ++t) {
          int e = p.e2p[r * p.topk + t];
          e = e < 0 ? 0 : (e >= p.num_perm ? p.num_perm - 1 : e);
          if (p.num_perm > 0) prefetch_l2(p.gemm2 + static_cast<size_t>(e) * H + h0);
        }
      }
    }
  }

  if (warp == 1 && lane < 3) {  // the mixes' first lines: L2 and address translation warm before the wait
    const float* mp = lane == 0 ? p.post : (lane == 1 ? p.comb : p.pre);
    if (mp != nullptr) prefetch_l2(mp);
  }
  // ---- 3. wait for the preceding kernel, let the next one launch, and read
  if (staged && !p.do_coeff) __syncthreads();  // the staged-rows barrier initialised
  griddep_wait();
  griddep_launch_dependents();
  PairLoads<N> cur;  // the row data first: the longest round trip goes out first
  if (staged) {
    if (tid == 0) {
      mbar_arrive_expect_tx(sbar, (p.P + N) * R * kCols * 2);
      tma_load_3d(const_cast<unsigned char*>(st_s), &tm_part, g * kCols, 0, 0, sbar);
      tma_load_3d(const_cast<unsigned char*>(st_s) + p.P * R * kCols * 2, &tm_res, g * kCols, 0, 0, sbar);
    }
  } else if (FRONT != kMoe && warp < npairs) {
    load_pair<N, FRONT>(p, warp * 2 + rq, h0, e2p_s, cur);
  }
  for (int k = tid; k < R * MIX; k += kT1) {  // [R][post n | comb n*n | pre n]
    const int r = k / MIX, c = k - r * MIX;
    if (c < N + N * N) {
      if (FRONT == kStreams || FRONT == kBroadcast) {
        mix_s[k] = 0.f;
      } else if (c < N) {
        cp_async4(mix_s + k, p.post + r * N + c);
      } else {
        cp_async4(mix_s + k, p.comb + r * N * N + (c - N));
      }
    } else if (p.pre != nullptr) {
      cp_async4(mix_s + k, p.pre + r * N + (c - N - N * N));
    } else {
      mix_s[k] = 0.f;
    }
  }
  if (FRONT == kMoe) {
    for (int k = tid; k < R * p.topk; k += kT1) {
      cp_async4(e2p_s + k, p.e2p + k);
      cp_async4(ew_s + k, p.ew + k);
    }
  }
  if (p.do_coeff && !packed) {
    // Split the fn slice into three bf16 terms (split3), stored column-major for
    // the MMA's B operand, while the row data and the mixes are in flight: a
    // thread takes 8 consecutive K values k = 8*oct .. 8*oct + 7 of column c (one
    // landed piece), consecutive threads consecutive columns, and writes each
    // term's 16 bytes at once.
    const bool ok = mbar_wait_bounded(bar, 0, deadline);
    if (!ok) record_error(status, MHC_ERR_DEVICE_TIMEOUT);
    if (__syncthreads_or(!ok)) {  // every copy issued has landed or never will
      cp_async_wait_all();
      return;
    }
    for (int e = tid; e < CP8 * (KC / 8); e += kT1) {
      const int c = e % CP8, oct = e / CP8;
      const float* src = reinterpret_cast<const float*>(fn_s + oct * PIECE) + c;  // k = 8*oct + i at src[i * C]
      unsigned w[3][4];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float f0 = c < C ? src[i * C] : 0.f, f1 = c < C ? src[(i + 1) * C] : 0.f;
        __nv_bfloat16 t0[3], t1[3];
        split3(f0, t0[0], t0[1], t0[2]);
        split3(f1, t1[0], t1[1], t1[2]);
#pragma unroll
        for (int t = 0; t < 3; ++t)
          w[t][i / 2] = static_cast<unsigned>(__bfloat16_as_ushort(t0[t])) |
                        (static_cast<unsigned>(__bfloat16_as_ushort(t1[t])) << 16);
      }
#pragma unroll
      for (int t = 0; t < 3; ++t)
        *reinterpret_cast<uint4*>(bs_s + (t * CP8 + c) * KS + oct * 8) = make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (FRONT == kMoe && warp < npairs) load_pair<N, FRONT>(p, warp * 2 + rq, h0, e2p_s, cur);
  if (staged) {  // one row pair per warp (rows <= 32): its vectors from the staged rows
    if (!mbar_wait_bounded(sbar, 0, deadline)) record_error(status, MHC_ERR_DEVICE_TIMEOUT);
    const int r = warp * 2 + rq;
    if (warp < npairs && r < R) {
#pragma unroll
      for (int j = 0; j < N; ++j)
        cur.rv[j] = *reinterpret_cast<const uint2*>(st_s + p.P * R * kCols * 2 + ((r * N + j) * kCols + vec * 4) * 2);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < p.P) cur.pv[u] = *reinterpret_cast<const uint2*>(st_s + ((u * R + r) * kCols + vec * 4) * 2);
    }
  }

  // ---- 4. row pairs: sum / finalize, post-mix, store the streams, sum c^2
  for (int q = warp; q < npairs; q += kW1) {
    PairLoads<N> nxt;
    if (q + kW1 < npairs) load_pair<N, FRONT>(p, (q + kW1) * 2 + rq, h0, e2p_s, nxt);
    const int r = q * 2 + rq;
    const bool valid = r < R;
    const float* mix = mix_s + (valid ? r : 0) * MIX;
    // Pairs of columns in packed f32x2 arithmetic (each element the same fp32
    // operations, in the same order, as one at a time).
    float2 nf[N][2];  // the new streams, as rounded to bf16
    uint2 nb[N];
    float2 xs[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) xs[t] = make_float2(0.f, 0.f);
    if (sums_partials(FRONT) || FRONT == kMoe) {
      float2 rf[N][2];
      if (valid) {
#pragma unroll
        for (int j = 0; j < N; ++j) unpack4x2(cur.rv[j], rf[j]);
        if (sums_partials(FRONT)) {
          const size_t off = static_cast<size_t>(r) * H + h0;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (u < p.P) {
              if (FRONT == kMailbox) cur.pv[u] = settle_slot(p.pptr[u] + off, cur.pv[u], deadline, status);
              float2 f[2];
              unpack4x2(cur.pv[u], f);
#pragma unroll
              for (int t = 0; t < 2; ++t) xs[t] = __fadd2_rn(xs[t], f[t]);
            }
          }
          for (int u = 8; u < p.P; ++u) {  // partials beyond the first 8
            float2 f[2];
            const __nv_bfloat16* src = p.pptr[u] + off;
            uint2 v = (FRONT == kMailbox || p.premote) ? ld_cg_v2(src) : ld_nc_v2(src);
            if (FRONT == kMailbox) v = settle_slot(src, v, deadline, status);
            unpack4x2(v, f);
#pragma unroll
            for (int t = 0; t < 2; ++t) xs[t] = __fadd2_rn(xs[t], f[t]);
          }
          if (FRONT == kMailbox) {  // consumed: back to "not written" for the round after next
            for (int u = 0; u < p.P; ++u)
              st_v2(const_cast<__nv_bfloat16*>(p.pptr[u]) + off, make_uint2(kNegZero2, kNegZero2));
          }
        } else {
          unpack4x2(cur.sv, xs);
          const int* idx = e2p_s + r * p.topk;
          const float* wt = ew_s + r * p.topk;
#pragma unroll
          for (int u = 0; u < 8; ++u) {  // the first 8 slots, loaded ahead
            if (u < p.topk) {
              const int e = idx[u];
              if (e >= p.num_perm) {
                if (vec == 0) record_error(status, MHC_ERR_DEVICE_INDEX);
              } else if (e >= 0) {
                float2 f[2];
                unpack4x2(cur.pv[u], f);
                const float2 w2 = make_float2(wt[u], wt[u]);
#pragma unroll
                for (int t = 0; t < 2; ++t) xs[t] = __ffma2_rn(w2, f[t], xs[t]);
              }
            }
          }
          for (int u = 8; u < p.topk; ++u) {  // slots beyond 8
            const int e = idx[u];
            if (e >= p.num_perm) {
              if (vec == 0) record_error(status, MHC_ERR_DEVICE_INDEX);
            } else if (e >= 0) {
              float2 f[2];
              unpack4x2(ld_nc_v2(p.gemm2 + static_cast<size_t>(e) * H + h0), f);
              const float2 w2 = make_float2(wt[u], wt[u]);
#pragma unroll
              for (int t = 0; t < 2; ++t) xs[t] = __ffma2_rn(w2, f[t], xs[t]);
            }
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < N; ++j)
#pragma unroll
          for (int t = 0; t < 2; ++t) rf[j][t] = make_float2(0.f, 0.f);
      }
      // mHC post: new[i] = bf16(post[i] * x + sum_j comb[j][i] * res[j])
#pragma unroll
      for (int i = 0; i < N; ++i) {
        float2 a[2];
        const float2 po = make_float2(mix[i], mix[i]);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          float2 s2 = __fmul2_rn(po, xs[t]);
#pragma unroll
          for (int j = 0; j < N; ++j) {
            const float cj = mix[N + j * N + i];
            s2 = __ffma2_rn(make_float2(cj, cj), rf[j][t], s2);
          }
          a[t] = s2;
        }
        nb[i] = make_uint2(pack_bf16x2(a[0].x, a[0].y), pack_bf16x2(a[1].x, a[1].y));
        unpack4x2(nb[i], nf[i]);
      }
    } else if (FRONT == kStreams) {
#pragma unroll
      for (int j = 0; j < N; ++j) {
        nb[j] = valid ? cur.rv[j] : make_uint2(0, 0);
        unpack4x2(nb[j], nf[j]);
      }
    } else {  // kBroadcast: every stream is the embedding row
      const uint2 xv = valid ? cur.sv : make_uint2(0, 0);
      unpack4x2(xv, xs);
#pragma unroll
      for (int j = 0; j < N; ++j) {
        nb[j] = xv;
#pragma unroll
        for (int t = 0; t < 2; ++t) nf[j][t] = xs[t];
      }
    }
    if (p.write_res && valid) {
#pragma unroll
      for (int i = 0; i < N; ++i) st_v2(p.residual_out + (static_cast<size_t>(r) * N + i) * H + h0, nb[i]);
    }
    if (p.aux_out != nullptr && valid) {  // mean over the streams, in stream order, rounded once
      constexpr float kInvN = 1.f / N;    // exact: n is a power of two
      uint2 ab;
      unsigned* aw = reinterpret_cast<unsigned*>(&ab);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        float2 m = nf[0][t];
#pragma unroll
        for (int j = 1; j < N; ++j) m = __fadd2_rn(m, nf[j][t]);
        m = __fmul2_rn(m, make_float2(kInvN, kInvN));
        aw[t] = pack_bf16x2(m.x, m.y);
      }
      st_v2(p.aux_out + static_cast<size_t>(r) * H + h0, ab);
    }
    if (p.do_layer) {  // collapse with the carried pre (identity pre-mix for the broadcast)
      float2 sq = make_float2(0.f, 0.f);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        float2 c;
        if (FRONT == kBroadcast) {
          c = xs[t];
        } else {
          c = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < N; ++j) {
            const float pj = mix[N + N * N + j];
            c = __ffma2_rn(make_float2(pj, pj), nf[j][t], c);
          }
        }
        sq = __ffma2_rn(c, c, sq);
      }
      const float sc2 = sum16_lanes(sq.x + sq.y);
      if (valid && vec == 0) p.sc2_part[r * G + g] = sc2;
    }
    if (p.do_coeff) {  // stage the streams for the projection; sum v^2 of the row
      float2 sv = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < N; ++i)
#pragma unroll
        for (int t = 0; t < 2; ++t) sv = __ffma2_rn(nf[i][t], nf[i][t], sv);
      const float sv2 = sum16_lanes(sv.x + sv.y);
      if (valid) {
#pragma unroll
        for (int i = 0; i < N; ++i) *reinterpret_cast<uint2*>(v_s + r * KS + i * kCols + vec * 4) = nb[i];
        if (vec == 0) p.dot_part[(static_cast<size_t>(r) * G + g) * RED + C] = sv2;
      }
    }
    cur = nxt;
  }
  if (!p.do_coeff) return;

  // ---- 5. projection of this block's n*64 stream values per row onto the C fn
  // columns on the tensor cores: [rows x n*64] bf16 x [n*64 x C] as three bf16
  // terms, fp32 accumulation (mma.sync m16n8k16).
  if (packed) {  // the packed slice, copied before the wait, has surely landed by now
    const bool ok = mbar_wait_bounded(bar, 0, deadline);
    if (!ok) record_error(status, MHC_ERR_DEVICE_TIMEOUT);
    if (__syncthreads_or(!ok)) return;  // also the barrier for the staged streams
  } else {
    __syncthreads();  // staged streams
  }
  // PAIRED (four row tiles or more): items are pairs of row tiles, so each B
  // fragment serves both tiles and the operand reads from shared memory, which
  // bound the projection with one tile per item, fall by ~30% (19.5 against
  // 20.2 us per boundary at 128 rows, 10.74 against 10.90 at 64). The single-tile
  // instantiation keeps the smaller kernel that fewer rows run faster with
  // (with both loops in one kernel: 7.82 against 7.76 us at 32 rows). Per
  // element the same operations in the same order either way.
  const int mtiles = (R + 15) >> 4;
  int mt0 = 0;  // first tile of the single-tile loop
  if constexpr (PAIRED) {
    const int mpairs = mtiles >> 1;
    mt0 = 2 * mpairs;  // an odd last tile goes to the single-tile loop
    for (int item = warp; item < mpairs * NT; item += kW1) {
      const int mp = item / NT, nt = item - mp * NT;
      float acc[2][3][4];
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int sp = 0; sp < 3; ++sp)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[t][sp][q] = 0.f;
      const __nv_bfloat16* arow = v_s + (mp * 32 + (lane & 15)) * KS + (lane >> 4) * 8;
      const __nv_bfloat16* brow = bs_s + (nt * 8 + (lane & 7)) * KS + ((lane >> 3) & 1) * 8;
#pragma unroll 2
      for (int k0 = 0; k0 < KC; k0 += 16) {
        unsigned a0[4], a1[4], b[3][2];
        ldmatrix_x4(a0, arow + k0);
        ldmatrix_x4(a1, arow + 16 * KS + k0);
#pragma unroll
        for (int sp = 0; sp < 3; ++sp) ldmatrix_x2(b[sp], brow + sp * CP8 * KS + k0);
#pragma unroll
        for (int sp = 0; sp < 3; ++sp) {
          mma_bf16_16816(acc[0][sp], a0, b[sp]);
          mma_bf16_16816(acc[1][sp], a1, b[sp]);
        }
      }
      const int col = nt * 8 + 2 * (lane & 3);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = (2 * mp + t) * 16 + (lane >> 2) + 8 * h;
          if (r < R && col < C) {
            float* dst = p.dot_part + (static_cast<size_t>(r) * G + g) * RED + col;
            dst[0] = (acc[t][0][2 * h] + acc[t][1][2 * h]) + acc[t][2][2 * h];
            if (col + 1 < C) dst[1] = (acc[t][0][2 * h + 1] + acc[t][1][2 * h + 1]) + acc[t][2][2 * h + 1];
          }
        }
      }
    }
  }
  // Single-tile items: (16-row tile, 8-column tile) of the block's rows x C
  // logits. A warp takes items w, w + 16, ...; for its item it runs every k-step, with
  // one accumulator per bf16 term of fn (three independent MMA chains), adds
  // the terms and stores its rows' dot products itself: no cross-warp sums.
  for (int item = warp; item < (mtiles - mt0) * NT; item += kW1) {
    const int mt = mt0 + item / NT, nt = item % NT;
    float acc[3][4];
#pragma unroll
    for (int sp = 0; sp < 3; ++sp)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[sp][q] = 0.f;
    const __nv_bfloat16* arow = v_s + (mt * 16 + (lane & 15)) * KS + (lane >> 4) * 8;
    const __nv_bfloat16* brow = bs_s + (nt * 8 + (lane & 7)) * KS + ((lane >> 3) & 1) * 8;
#pragma unroll 4
    for (int k0 = 0; k0 < KC; k0 += 16) {
      unsigned a[4], b[3][2];
      ldmatrix_x4(a, arow + k0);
#pragma unroll
      for (int sp = 0; sp < 3; ++sp) ldmatrix_x2(b[sp], brow + sp * CP8 * KS + k0);
#pragma unroll
      for (int sp = 0; sp < 3; ++sp) mma_bf16_16816(acc[sp], a, b[sp]);
    }
    // C fragment: lane holds rows lane/4 and lane/4 + 8, columns 2*(lane%4) + {0, 1}
    const int col = nt * 8 + 2 * (lane & 3);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = mt * 16 + (lane >> 2) + 8 * h;
      if (r < R && col < C) {
        float* dst = p.dot_part + (static_cast<size_t>(r) * G + g) * RED + col;
        dst[0] = (acc[0][2 * h] + acc[1][2 * h]) + acc[2][2 * h];
        if (col + 1 < C) dst[1] = (acc[0][2 * h + 1] + acc[1][2 * h + 1]) + acc[2][2 * h + 1];
      }
    }
  }
}

// Sinkhorn normalisation of an n x n matrix in one thread's registers: `iters`
// times, each row divided by (its sum + eps), then each column by (its sum +
// eps). For n = 4 the matrix stays as it came, K, and the steps update scale
// vectors, M = diag(a) K diag(b): a row step's denominator is a_j (K b)_j + eps,
// so with al_j = 1 / a_j it becomes al_j <- (K b)_j + eps al_j and a_j = 1 / al_j
// (columns likewise with be = 1 / b). eps rides in the first fused multiply-add
// of each dot product, so a step is three dependent additions and a
// reciprocal, with 28 instructions against 36 for scaling the matrix in place
// (2,400 against 2,761 cycles for 20 iterations, measured on this part alone).
// Scalar code beats packed f32x2 pairs here, and neither sharing the matrix
// between lanes (a shuffle costs about 27 cycles) nor taking a step's four
// reciprocals from one (batch inversion) is faster.
// Each denominator also gets the smallest normal float, added off the chain: a
// row (or column) of K that is exactly zero (its logits some 100 or more below the
// largest) would otherwise shrink its denominator by eps every step until it
// underflows, and 1/0 times 0 is NaN where scaling in place gives 0. In fp32 the
// term changes nothing unless the denominator is already below ~2e-31.
constexpr float kTinyNormal = 1.17549435e-38f;  // 2^-126
template <int N>
__device__ __forceinline__ void sinkhorn_iterate(float (&M)[N][N], int iters, float eps) {
  if constexpr (N == 1) {
    for (int it = 0; it < iters; ++it) {
      M[0][0] *= rcp_approx(M[0][0] + eps);
      M[0][0] *= rcp_approx(M[0][0] + eps);
    }
  } else if constexpr (N == 2) {
    float2 P[2] = {make_float2(M[0][0], M[0][1]), make_float2(M[1][0], M[1][1])};
    const float2 e2 = make_float2(eps, eps);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float rr = rcp_approx(P[j].x + P[j].y + eps);
        P[j] = __fmul2_rn(P[j], make_float2(rr, rr));
      }
      const float2 c2 = __fadd2_rn(__fadd2_rn(P[0], P[1]), e2);
      const float2 r2 = make_float2(rcp_approx(c2.x), rcp_approx(c2.y));
      P[0] = __fmul2_rn(P[0], r2);
      P[1] = __fmul2_rn(P[1], r2);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      M[j][0] = P[j].x;
      M[j][1] = P[j].y;
    }
  } else {
    static_assert(N == 4, "hc_mult 1, 2 or 4");
    float a[4], b[4], al[4], be[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      a[k] = 1.f;
      b[k] = 1.f;
      al[k] = 1.f;
      be[k] = 1.f;
    }
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // rows: al_j <- (K b)_j + eps al_j
        const float q0 = fmaf(M[j][1], b[1], fmaf(M[j][0], b[0], fmaf(eps, al[j], kTinyNormal)));
        const float q1 = fmaf(M[j][3], b[3], M[j][2] * b[2]);
        al[j] = q0 + q1;
        a[j] = rcp_approx(al[j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // columns: be_i <- (K^T a)_i + eps be_i
        const float q0 = fmaf(M[1][i], a[1], fmaf(M[0][i], a[0], fmaf(eps, be[i], kTinyNormal)));
        const float q1 = fmaf(M[3][i], a[3], M[2][i] * a[2]);
        be[i] = q0 + q1;
        b[i] = rcp_approx(be[i]);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) M[j][i] = (a[j] * M[j][i]) * b[i];
  }
}

// Loads of one layer-input task of a lane (row r, 8 columns): the row's
// per-block sums of c^2, its carried pre, the stream vectors and norm weights.
template <int N>
struct LayerLoads {
  static constexpr int MAXM = (kMaxBlocks + 31) / 32;
  float sq[MAXM];
  float pr[N];
  uint4 sv[N];
  uint4 nw;
};

template <int N>
__device__ __forceinline__ void layer_load(const Params& p, int r, int g, int lane, bool weights,
                                           LayerLoads<N>& Q) {
  const int G = p.H / kCols;
#pragma unroll
  for (int m = 0; m < LayerLoads<N>::MAXM; ++m) {
    const int k = lane + 32 * m;
    Q.sq[m] = k < G ? __ldcg(p.sc2_part + r * G + k) : 0.f;
  }
  if (g >= G) return;
  const int h0 = g * kCols + (lane & 7) * 8;
  if (weights) Q.nw = ld_nc_v4(p.norm_weight + h0);
  if (p.tail_broadcast) {
    Q.sv[0] = ld_v4(p.tail_streams + static_cast<size_t>(r) * p.H + h0);
  } else {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      Q.pr[j] = p.pre[r * N + j];
      Q.sv[j] = ld_v4(p.tail_streams + (static_cast<size_t>(r) * N + j) * p.H + h0);
    }
  }
}

// The tail of a boundary, launched after the streaming kernel (programmatic
// dependent launch). Layer-input blocks split the rows into tasks of 256
// columns (4 units of 64), one task per warp at a time: a lane normalises 8
// columns of the row into the layer input (and MXFP8), recomputing the
// collapse from the bf16 streams, after summing the row's per-block c^2 itself.
// Coefficient blocks finish rows j, j + Gc, ... (logits, sigmoid, Sinkhorn).
template <int N>
__global__ void __launch_bounds__(kThreads, 2) boundary_tail_kernel(const Params p) {
  constexpr int C = logits_of(N);
  constexpr int RED = red_of(N);
  extern __shared__ __align__(128) unsigned char smem[];
  const TailLayout L = tail_layout<N>();
  float* slot_s = reinterpret_cast<float*>(smem + L.part_off);  // [kWarps rows][kWarps][RED]
  float* scale_s = reinterpret_cast<float*>(smem + L.cst_off);
  float* base_s = scale_s + 4;

  const int G = p.H / kCols;
  const int H = p.H;
  const int R = p.R;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rq = lane >> 3, vec = lane & 7;

  // block roles: coefficient blocks first or last in the grid (the first blocks
  // are placed first, on the SMs the streaming kernel leaves free)
  const int bid = blockIdx.x;
  const int lbid = p.tail_coeff_first ? bid - p.tail_coeff_blocks : bid;
  if (lbid >= 0 && lbid < p.tail_layer_blocks) {
    const int GT = (G + 3) >> 2;  // tasks per row
    const int T = R * GT;
    const int W = p.tail_layer_blocks * kWarps;
    const int w0 = lbid * kWarps + warp;
    LayerLoads<N> cur;
    if (w0 < T) {  // norm weights of the first task: weights, so before the wait
      const int g = (w0 % GT) * 4 + rq;
      if (g < G) cur.nw = ld_nc_v4(p.norm_weight + g * kCols + vec * 8);
      // lines the first task reads after the wait: L2 and address translation warm
      const int r = w0 / GT;
      if (lane == 0) prefetch_l2(p.sc2_part + r * G);
      if (lane == 1 && !p.tail_broadcast) prefetch_l2(p.pre + r * N);
      if (lane == 2) prefetch_l2(p.tail_streams + static_cast<size_t>(r) * (p.tail_broadcast ? 1 : N) * H);
    }
    griddep_wait();
    griddep_launch_dependents();
    if (w0 < T) layer_load<N>(p, w0 / GT, (w0 % GT) * 4 + rq, lane, false, cur);
    const int scols = H / 32;
    const int col_tiles = (scols + 3) / 4;
    for (int t = w0; t < T; t += W) {
      LayerLoads<N> nxt;
      if (t + W < T) layer_load<N>(p, (t + W) / GT, ((t + W) % GT) * 4 + rq, lane, true, nxt);
      const int r = t / GT;
      const int g = (t - r * GT) * 4 + rq;
      // ---- 7. the row's inverse RMS of the collapse: block sums in a fixed order
      float a = cur.sq[0];
#pragma unroll
      for (int m = 1; m < LayerLoads<N>::MAXM; ++m) a += cur.sq[m];
      a = warp_sum(a);
      const float inv = rsqrtf(__fdiv_rn(a, static_cast<float>(H)) + p.norm_eps);
      if (g < G) {  // the 8 lanes of a unit share g: whole MXFP8 groups
        const int h0 = g * kCols + vec * 8;
        // ---- 7b. layer input: the collapse recomputed from the bf16 streams exactly
        // as the streaming kernel summed its squares
        float c[8];
        if (p.tail_broadcast) {
          unpack8(cur.sv[0], c);
        } else {
          float nf[N][8];
#pragma unroll
          for (int j = 0; j < N; ++j) unpack8(cur.sv[j], nf[j]);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < N; ++j) s = fmaf(cur.pr[j], nf[j][e], s);
            c[e] = s;
          }
        }
        float w[8], y[8], yr[8];
        unpack8(cur.nw, w);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = c[e] * inv * w[e];
        const uint4 yb = round8(y, yr);
        st_v4(p.layer_input + static_cast<size_t>(r) * H + h0, yb);
        if (p.q_data != nullptr) {
          float amax = 0.f;
          bool finite = true;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            amax = fmaxf(amax, fabsf(yr[e]));
            finite = finite && isfinite(yr[e]);
          }
          // the 4 lanes of a 32-column block are vec 0-3 or 4-7 of the same unit
          const unsigned grp_mask = 0xffu << (lane & 24);
          amax = fmaxf(amax, __shfl_xor_sync(grp_mask, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(grp_mask, amax, 2));
          const unsigned fin_mask = __ballot_sync(grp_mask, finite);
          const unsigned grp = (fin_mask >> (lane & 28)) & 0xfu;
          uint2 d;
          unsigned char sbyte;
          if (grp == 0xfu) {
            const int e = e8m0_exponent(amax);
            const float sc = exp2_neg(e);
            d.x = static_cast<unsigned>(e4m3x2(yr[0] * sc, yr[1] * sc)) |
                  (static_cast<unsigned>(e4m3x2(yr[2] * sc, yr[3] * sc)) << 16);
            d.y = static_cast<unsigned>(e4m3x2(yr[4] * sc, yr[5] * sc)) |
                  (static_cast<unsigned>(e4m3x2(yr[6] * sc, yr[7] * sc)) << 16);
            sbyte = static_cast<unsigned char>(e + 127);
          } else {
            d.x = d.y = 0x7f7f7f7fu;
            sbyte = 0xff;
          }
          *reinterpret_cast<uint2*>(p.q_data + static_cast<size_t>(r) * H + h0) = d;
          if ((vec & 3) == 0) {
            const int sc = h0 / 32;
            const int off = p.q_swizzled ? swizzled_scale_offset(r, sc, col_tiles) : r * scols + sc;
            p.q_scale[off] = sbyte;
          }
        }
      }
      cur = nxt;
    }
    if (p.q_data != nullptr && p.q_swizzled) {
      // zero the padding of the swizzled scale buffer: rows R.. whole (4-byte words
      // of a tile row when the buffer is 4-byte aligned), then the padding columns
      // of rows below R
      const int rows_p = (R + 127) & ~127;
      const int pad_cols = col_tiles * 4 - scols;
      const bool words = (reinterpret_cast<uintptr_t>(p.q_scale) & 3) == 0;
      const int per_row = words ? col_tiles : col_tiles * 4;
      const int n_rows = (rows_p - R) * per_row;
      const int n_cols = R * pad_cols;
      for (int k = w0 * 32 + lane; k < n_rows + n_cols; k += W * 32) {
        if (k < n_rows) {
          const int r = R + k / per_row, u = k % per_row;
          if (words)
            *reinterpret_cast<uint32_t*>(p.q_scale + swizzled_scale_offset(r, u * 4, col_tiles)) = 0u;
          else
            p.q_scale[swizzled_scale_offset(r, u, col_tiles)] = 0;
        } else {
          const int kk = k - n_rows;
          const int r = kk / pad_cols, sc = scols + kk % pad_cols;
          p.q_scale[swizzled_scale_offset(r, sc, col_tiles)] = 0;
        }
      }
    }
  } else {
    // Coefficient rows jb, jb + CB, ...: in batches of up to kWarps rows, every
    // warp adds a share of each row's per-block records (fixed order) into a
    // slot, then warp s finishes row s of the batch: logits, sigmoid, Sinkhorn.
    const int jb = p.tail_coeff_first ? bid : bid - p.tail_layer_blocks;
    const int CB = p.tail_coeff_blocks;
    if (tid < 3) cp_async4(scale_s + tid, p.scale + tid);  // weights: before the wait
    if (tid >= 32 && tid < 32 + C) cp_async4(base_s + tid - 32, p.base + (tid - 32));
    if (tid == 64) prefetch_l2(p.dot_part + static_cast<size_t>(jb) * G * RED);  // warm, as above
    griddep_wait();
    griddep_launch_dependents();
    constexpr int V4 = RED / 4;
    constexpr int MAXK = (kMaxBlocks * V4 + kThreads - 1) / kThreads;
    constexpr int NN = N * N;
    const int F = G * V4;
    const int rho = (R - jb + CB - 1) / CB;
    cp_async_wait_all();
    for (int k0 = 0; k0 < rho; k0 += kWarps) {
      const int nk = rho - k0 < kWarps ? rho - k0 : kWarps;
      float4 v[MAXK];
      {
        const float4* base = reinterpret_cast<const float4*>(p.dot_part + static_cast<size_t>(jb + k0 * CB) * G * RED);
#pragma unroll
        for (int k = 0; k < MAXK; ++k) {
          const int f = tid + k * kThreads;
          v[k] = f < F ? __ldcg(base + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      for (int s = 0; s < nk; ++s) {
        float4 nx[MAXK];
        if (s + 1 < nk) {  // the next row's loads go out before this row is added up
          const float4* base =
              reinterpret_cast<const float4*>(p.dot_part + static_cast<size_t>(jb + (k0 + s + 1) * CB) * G * RED);
#pragma unroll
          for (int k = 0; k < MAXK; ++k) {
            const int f = tid + k * kThreads;
            nx[k] = f < F ? __ldcg(base + f) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float4 a = v[0];
#pragma unroll
        for (int k = 1; k < MAXK; ++k) {
          a.x += v[k].x;
          a.y += v[k].y;
          a.z += v[k].z;
          a.w += v[k].w;
        }
        // lanes sharing lane % V4 hold the same 4 record values: add them up
#pragma unroll
        for (int m = V4; m < 32; m <<= 1) {
          a.x += __shfl_xor_sync(kFull, a.x, m);
          a.y += __shfl_xor_sync(kFull, a.y, m);
          a.z += __shfl_xor_sync(kFull, a.z, m);
          a.w += __shfl_xor_sync(kFull, a.w, m);
        }
        if (lane < V4) reinterpret_cast<float4*>(slot_s + (s * kWarps + warp) * RED)[lane] = a;
        if (s + 1 < nk) {
#pragma unroll
          for (int k = 0; k < MAXK; ++k) v[k] = nx[k];
        }
      }
      __syncthreads();
      // warp s < nk: the comb (Sinkhorn) of row s of the batch; the pre and post of
      // row s go to warp s + nk where there is one, else warp s does them after
      const int s_comb = warp < nk ? warp : -1;
      const int s_pp = warp < nk ? (warp + nk < kWarps ? -1 : warp) : (warp - nk < nk ? warp - nk : -1);
      if (s_comb >= 0 || s_pp >= 0) {
        const int sl = s_comb >= 0 ? s_comb : s_pp;
        const int r = jb + (k0 + sl) * CB;
        float s = 0.f;  // lane c: record value c, the warps' shares added in order
        if (lane < RED) {
#pragma unroll
          for (int w = 0; w < kWarps; ++w) s += slot_s[(sl * kWarps + w) * RED + lane];
        }
        const float inv = rsqrtf(__fdiv_rn(__shfl_sync(kFull, s, C), static_cast<float>(N * H)) + p.rms_eps);
        const int grp = lane < N ? 0 : (lane < 2 * N ? 1 : 2);
        const float l = lane < C ? scale_s[grp] * inv * s + base_s[lane] : 0.f;
        if (s_comb >= 0) {
          // M = exp(L - max L) with one exp per lane, then Sinkhorn in one thread
          float lk = __shfl_sync(kFull, l, (lane + 2 * N) & 31);  // lane k < n*n: comb logit k
          const float mx = warp_max(lane < NN ? lk : -INFINITY);
          const float ek = expf(lk - mx);
          float lc[NN];
#pragma unroll
          for (int k = 0; k < NN; ++k) lc[k] = __shfl_sync(kFull, ek, k);
          if (lane == 0) {
            float M[N][N];
#pragma unroll
            for (int j = 0; j < N; ++j)
#pragma unroll
              for (int i = 0; i < N; ++i) M[j][i] = lc[j * N + i];
            sinkhorn_iterate<N>(M, p.iters, p.sk_eps);
#pragma unroll
            for (int j = 0; j < N; ++j)
#pragma unroll
              for (int i = 0; i < N; ++i) p.comb_out[r * NN + j * N + i] = M[j][i];
          }
        }
        if (s_pp >= 0) {
          if (lane < N) {
            p.pre_out[r * N + lane] = 1.f / (1.f + expf(-l)) + p.pre_eps;
          } else if (lane < 2 * N) {
            p.post_out[r * N + (lane - N)] = p.alpha / (1.f + expf(-l));
          }
        }
      }
      __syncthreads();  // the slots are refilled by the next batch
    }
  }
}


// Mailbox of a consumer (one per rank of a TP group, in that rank's memory):
// a 256-byte header (the status word at byte 0, the consumed round + 1 per parity
// at bytes 8 and 12), then the slots [2 parities][W producers][M rows][H] bf16,
// M the mailbox's row capacity. A slot element that holds negative zero has not
// been written yet: the consumer turns every element it reads back into that
// mark, and a producer never stores it.
constexpr size_t kMailboxHeader = 256;

inline size_t mailbox_total(int W, int M, int H) {
  return kMailboxHeader + static_cast<size_t>(2) * W * M * H * 2;
}

struct PublishParams {
  unsigned char* mb[kMaxPartials];  // every consumer's mailbox (this GPU's or a peer's)
  const __nv_bfloat16* x;           // this producer's contribution [R, H]
  unsigned* status;                 // this producer's own mailbox header
  int rank, W, M, H;
  unsigned round;
  int64_t budget_ns;
};

// Producer side: block (r, c) stores row r of x, negative zeros made positive,
// into slot [parity][rank][r] of consumer c's mailbox once c has consumed the
// round that last used this parity (bounded wait). No flag follows: each element
// is its own mark, so nothing waits for the stores to be acknowledged.
__global__ void __launch_bounds__(256) mailbox_publish_kernel(const PublishParams q) {
  const int r = blockIdx.x, c = blockIdx.y;
  const unsigned par = q.round & 1u;
  unsigned char* mb = q.mb[c];
  const unsigned* done = reinterpret_cast<const unsigned*>(mb + 8);
  bool ok = true;
  if (threadIdx.x == 0) {
    const long long deadline = wait_deadline(q.budget_ns);
    while (ok && ld_acquire_sys(done + par) + 1u < q.round) ok = clock64() <= deadline;
    if (!ok) record_error(q.status, MHC_ERR_DEVICE_TIMEOUT);
  }
  // the barrier carries thread 0's acquire to every thread's stores
  if (__syncthreads_or(!ok)) return;  // nothing written for a consumer that is behind
  __nv_bfloat16* slot = reinterpret_cast<__nv_bfloat16*>(mb + kMailboxHeader) +
                        ((static_cast<size_t>(par) * q.W + q.rank) * q.M + r) * q.H;
  const __nv_bfloat16* src = q.x + static_cast<size_t>(r) * q.H;
  mailbox_store_row(slot, src, q.H, threadIdx.x, blockDim.x);
}

// After a collect: the round is consumed, its parity's slots may be reused. If
// the collect recorded an error (a slot wait that ran out: the slots it gave up
// on were neither summed nor re-marked), the round stays unconsumed, so that a
// producer's next publish into this parity runs out of its own wait and reports
// it instead of the stale slots passing for fresh ones.
__global__ void mailbox_done_kernel(unsigned* done, unsigned par, unsigned value, const unsigned* ws_status) {
  if (ws_status != nullptr && ld_acquire_gpu(ws_status) != 0u) return;
  __threadfence_system();
  st_release_sys(done + par, value);
}

// A fresh mailbox: header zero, every slot element negative zero.
__global__ void mailbox_init_kernel(unsigned char* mb, size_t units) {
  const size_t i0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i0 < kMailboxHeader / 16) st_v4(mb + i0 * 16, make_uint4(0, 0, 0, 0));
  const uint4 z = make_uint4(kNegZero2, kNegZero2, kNegZero2, kNegZero2);
  for (size_t i = i0; i < units; i += static_cast<size_t>(gridDim.x) * blockDim.x)
    st_v4(mb + kMailboxHeader + i * 16, z);
}

// fn [n*H, C] fp32 -> per block g the B operand of its projection as three bf16
// terms, [G][3][CP8][n*64 + 8]: entry (t, c, k) is term t of fn[(k/64)*H + 64g + k%64][c];
// columns c >= C and the 8-entry gap after each column are zero.
template <int N>
__global__ void __launch_bounds__(256) pack_projection_kernel(const float* __restrict__ fn, int H,
                                                              __nv_bfloat16* __restrict__ out) {
  constexpr int C = logits_of(N);
  constexpr int KS = kstride_of(N);
  constexpr int CP8 = ntiles_of(N) * 8;
  const int g = blockIdx.x;
  __nv_bfloat16* dst = out + static_cast<size_t>(g) * (packed_slice_bytes(N) / 2);
  for (int e = threadIdx.x; e < CP8 * KS; e += blockDim.x) {
    const int c = e / KS, k = e - c * KS;
    float f = 0.f;
    if (c < C && k < N * kCols) f = fn[(static_cast<size_t>(k / kCols) * H + g * kCols + k % kCols) * C + c];
    __nv_bfloat16 hi, mid, lo;
    split3(f, hi, mid, lo);
    dst[(0 * CP8 + c) * KS + k] = hi;
    dst[(1 * CP8 + c) * KS + k] = mid;
    dst[(2 * CP8 + c) * KS + k] = lo;
  }
}

// MXFP8 of a bf16 [R, H] matrix: a lane quantises 8 columns, 4 lanes a block.
__global__ void __launch_bounds__(256) mxfp8_rows_kernel(const __nv_bfloat16* __restrict__ x, int R, int H,
                                                          uint8_t* __restrict__ data, uint8_t* __restrict__ scale,
                                                          int swizzled) {
  griddep_wait();
  griddep_launch_dependents();
  const int lanes_per_row = H / 8;
  const int scols = H / 32;
  const int col_tiles = (scols + 3) / 4;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(R) * lanes_per_row;
  const int lane = threadIdx.x & 31;
  // lanes_per_row is a multiple of 4 and blockDim a multiple of 32: a block's 4
  // lanes are always in the same warp and either all active or all idle
  const bool active = gid < total;
  const int r = active ? static_cast<int>(gid / lanes_per_row) : 0;
  const int h0 = active ? static_cast<int>(gid - static_cast<long long>(r) * lanes_per_row) * 8 : 0;
  float y[8];
  if (active) {
    unpack8(ld_nc_v4(x + static_cast<size_t>(r) * H + h0), y);
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) y[t] = 0.f;
  }
  float amax = 0.f;
  bool finite = true;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    amax = fmaxf(amax, fabsf(y[t]));
    finite = finite && isfinite(y[t]);
  }
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
  const unsigned fin_mask = __ballot_sync(kFull, finite);
  if (!active) return;
  const unsigned grp = (fin_mask >> (lane & 28)) & 0xfu;
  uint2 d;
  unsigned char sbyte;
  if (grp == 0xfu) {
    const int e = e8m0_exponent(amax);
    const float s = exp2_neg(e);
    d.x = static_cast<unsigned>(e4m3x2(y[0] * s, y[1] * s)) | (static_cast<unsigned>(e4m3x2(y[2] * s, y[3] * s)) << 16);
    d.y = static_cast<unsigned>(e4m3x2(y[4] * s, y[5] * s)) | (static_cast<unsigned>(e4m3x2(y[6] * s, y[7] * s)) << 16);
    sbyte = static_cast<unsigned char>(e + 127);
  } else {
    d.x = d.y = 0x7f7f7f7fu;
    sbyte = 0xff;
  }
  *reinterpret_cast<uint2*>(data + static_cast<size_t>(r) * H + h0) = d;
  if (((h0 / 8) & 3) == 0) {
    const int sc = h0 / 32;
    scale[swizzled ? swizzled_scale_offset(r, sc, col_tiles) : r * scols + sc] = sbyte;
  }
}

// Zero the padding bytes of a swizzled scale buffer (rows >= R or columns >= H/32).
__global__ void scale_padding_kernel(uint8_t* scale, int R, int H) {
  griddep_wait();
  griddep_launch_dependents();
  const int scols = H / 32;
  const int col_tiles = (scols + 3) / 4;
  const int rows_p = (R + 127) & ~127;
  const int cols_p = col_tiles * 4;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < rows_p * cols_p; k += gridDim.x * blockDim.x) {
    const int r = k / cols_p, c = k - r * cols_p;
    if (r >= R || c >= scols) scale[swizzled_scale_offset(r, c, col_tiles)] = 0;
  }
}

}  // namespace mhc

// =====================================================================================
// Host side: argument checks, launch configuration, C ABI
// =====================================================================================

namespace {

using namespace mhc;

int64_t g_budget_ns = 1000000000LL;
int g_extra_tx = 0;

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t ws_layout(int R, int H, int n, size_t* sc2_off, size_t* dot_off) {
  const int G = H / kCols;
  const size_t a = kWsHeader;
  const size_t sc2 = (static_cast<size_t>(R) * G * 4 + 255) & ~static_cast<size_t>(255);
  const size_t dot = static_cast<size_t>(R) * G * red_of(n) * 4;
  if (sc2_off) *sc2_off = a;
  if (dot_off) *dot_off = a + sc2;
  return a + sc2 + dot;
}

bool shape_ok(int R, int H, int n) {
  return R >= 1 && R <= kMaxRows && H >= kCols && H % kCols == 0 && H / kCols <= kMaxBlocks &&
         (n == 1 || n == 2 || n == 4);
}

mhc_status check_coeff(const mhc_coeff_args* a) {
  if (a == nullptr) return MHC_OK;
  if ((!a->fn && !a->fn_packed) || !a->scale || !a->base) return MHC_ERR_INVALID_ARG;
  if (!aligned(a->fn, 16) || !aligned(a->fn_packed, 16) || !aligned(a->scale, 4) || !aligned(a->base, 4))
    return MHC_ERR_INVALID_ARG;
  if (!(a->rms_eps >= 0.f) || !(a->pre_eps >= 0.f) || !(a->sinkhorn_eps >= 0.f)) return MHC_ERR_INVALID_ARG;
  if (a->sinkhorn_iters < 0 || a->sinkhorn_iters > kMaxIters) return MHC_ERR_INVALID_ARG;
  return MHC_OK;
}

mhc_status check_mxfp8(const mhc_mxfp8_out* q) {
  if (q == nullptr) return MHC_OK;
  if (!q->data || !q->scale || !aligned(q->data, 8)) return MHC_ERR_INVALID_ARG;
  return MHC_OK;
}

// Launch with programmatic stream serialization: the kernel may start while the
// preceding kernel on the stream finishes, and waits for it (griddepcontrol.wait)
// before reading anything that kernel may have written.
// A carveout >= 0 sets this launch's preferred shared-memory share (percent).
template <typename Kern, typename... Extra>
mhc_status launch_pdl(Kern kern, int grid, int smem, cudaStream_t stream, const Params& p, int threads = kThreads,
                      int carveout = -1, const Extra&... extra) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (carveout >= 0) {
    attr[1].id = cudaLaunchAttributePreferredSharedMemoryCarveout;
    attr[1].val.sharedMemCarveout = static_cast<unsigned>(carveout);
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, kern, p, extra...) != cudaSuccess) {
    (void)cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  return MHC_OK;
}

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

// A 3-D bf16 tensor map (innermost dimension first; strides in bytes of
// dimensions 1 and 2), no swizzle, out-of-range elements read as zero.
bool make_map3(CUtensorMap* m, const void* base, const uint64_t (&dims)[3], const uint64_t (&strides)[2],
               const uint32_t (&box)[3]) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]}, st[2] = {strides[0], strides[1]};
  cuuint32_t b[3] = {box[0], box[1], box[2]}, e[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), d, st, b, e,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor maps of the staged rows (partials front, this GPU's memory): the P
// partials as a [P][R][H] box {64, R, P} (uniform positive stride between
// partials) and the streams [R][n][H] as a box {64, n, R}. False when the call
// does not qualify or a map cannot be made; the kernel then loads per lane.
template <int N>
bool staged_maps(const Params& p, CUtensorMap* maps) {
  if (p.premote || p.R > kStagedRows || p.P > 8) return false;
  const int64_t stride = p.P > 1 ? static_cast<int64_t>(p.pptr[1] - p.pptr[0]) : static_cast<int64_t>(p.R) * p.H;
  if (stride <= 0 || stride % 8 != 0) return false;
  for (int u = 2; u < p.P; ++u)
    if (static_cast<int64_t>(p.pptr[u] - p.pptr[0]) != u * stride) return false;
  const uint64_t H = static_cast<uint64_t>(p.H), R = static_cast<uint64_t>(p.R);
  const uint64_t pd[3] = {H, R, static_cast<uint64_t>(p.P)}, ps[2] = {H * 2, static_cast<uint64_t>(stride) * 2};
  const uint32_t pb[3] = {kCols, static_cast<uint32_t>(R), static_cast<uint32_t>(p.P)};
  const uint64_t rd[3] = {H, static_cast<uint64_t>(N), R}, rs[2] = {H * 2, H * 2 * N};
  const uint32_t rb[3] = {kCols, static_cast<uint32_t>(N), static_cast<uint32_t>(R)};
  return make_map3(&maps[0], p.pptr[0], pd, ps, pb) && make_map3(&maps[1], p.residual, rd, rs, rb);
}

// Number of SMs of the current device (cached per device; safe to call from
// several host threads).
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kMaxBlocks;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return kMaxBlocks;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Raise a kernel's dynamic shared memory limit to 200 KB, once per device
// (idempotent, so concurrent first calls only repeat the same setting).
constexpr int kSmemLimit = 200 * 1024;

// Placement of the tail's blocks. An SM changes its L1 / shared-memory split only
// when it is empty, and the split the driver picks for the streaming kernel alone
// (just above its shared memory) leaves no room for a tail block beside it. Up to
// kCoexistRows rows the streaming kernel asks for the largest shared-memory split,
// so tail blocks launch early on its SMs too, and from kCoeffFirstRows rows the
// coefficient blocks take the first block indices, which land on the SMs the
// streaming kernel leaves free. Measured on B200 (whole boundaries in CUDA graphs,
// us per boundary): 7.84 against 8.26 at 32 rows, 6.84 against 7.05 at 16, 5.85
// against 5.94 at 4; the largest split is slower from 48 rows on (10.23 against
// 9.95 at 48, 11.6 against 10.9 at 64, 22.2 against 19.9 at 128), and at 2 rows
// the coefficient blocks first are (6.20 against 6.07). The coefficient blocks
// stay first up to kCoeffFirstMaxRows rows, without the largest split: 9.31 /
// 9.64 / 10.09 / 10.73 / 12.95 against 9.53 / 9.82 / 10.59 / 11.04 / 13.15 at
// 40 / 48 / 56 / 64 / 80 rows; from 96 rows on they are better last (14.07 /
// 16.16 against 14.26 / 16.30 at 96 / 128).
constexpr int kCoexistRows = 32;
constexpr int kCoeffFirstRows = 4;
constexpr int kCoeffFirstMaxRows = 80;
template <typename Kern>
bool allow_smem(Kern kern, int bytes, std::atomic<int>* configured) {
  int dev = 0;
  if (bytes > kSmemLimit || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (configured[dev].load(std::memory_order_acquire) != 0) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  configured[dev].store(1, std::memory_order_release);
  return true;
}

template <int N, int FRONT>
mhc_status launch_boundary(Params& p, cudaStream_t stream) {
  CUtensorMap maps[2];
  std::memset(maps, 0, sizeof(maps));
  p.staged = FRONT == kPartials && staged_maps<N>(p, maps) ? 1 : 0;
  const SmemLayout L = smem_layout<N>(p.R, p.topk, FRONT == kMoe, p.fn_packed != nullptr, p.staged ? p.P : 0);
  static std::atomic<int> configured[2][64];
  const bool paired = ((p.R + 15) >> 4) >= 4;
  auto kern = paired ? boundary_kernel<N, FRONT, true> : boundary_kernel<N, FRONT, false>;
  if (!allow_smem(kern, L.total, configured[paired ? 1 : 0])) return MHC_ERR_CUDA;
  p.extra_tx = g_extra_tx;
  p.budget_ns = g_budget_ns;
  const int G = p.H / kCols;
  const bool few_rows = p.R <= kCoexistRows;
  mhc_status st = launch_pdl(kern, G, L.total, stream, p, kT1,
                             few_rows ? static_cast<int>(cudaSharedmemCarveoutMaxShared) : -1, maps[0], maps[1]);
  if (st != MHC_OK || !(p.do_layer || p.do_coeff)) return st;
  if (FRONT == kBroadcast) {
    p.tail_streams = p.x;
    p.tail_broadcast = 1;
  } else {
    p.tail_streams = FRONT == kStreams ? p.residual : p.residual_out;
    p.tail_broadcast = 0;
  }
  // Coefficient blocks: as many as the SMs that G layer-input blocks leave (at
  // most one per row), and at least one for every two rows (a block takes its
  // rows' records one after the other: 14.02 / 14.53 us per boundary at 96 rows,
  // 16.19 / 16.81 at 128 against the free SMs alone; one block per row, 17.31 at
  // 128). Layer-input blocks: one 256-column task per warp, as many blocks as fill
  // the SMs twice (the tail runs two blocks an SM) beside the coefficient
  // blocks; up to G of them start beside the streaming kernel, the rest as its
  // blocks retire. Against at most G layer-input blocks (B200, us per boundary):
  // 10.92 / 11.12 at 64 rows, 14.34 / 15.53 at 96, 16.93 / 18.20 at 128.
  const int tasks = p.R * ((G + 3) / 4);
  const int lb = (tasks + kWarps - 1) / kWarps;
  const int spare = sm_count() - (p.do_layer ? (lb < G ? lb : G) : 0);
  p.tail_coeff_blocks = p.do_coeff ? (p.R < spare ? p.R : (spare > 1 ? spare : 1)) : 0;
  if (p.do_coeff && p.tail_coeff_blocks < (p.R + 1) / 2) p.tail_coeff_blocks = (p.R + 1) / 2;
  // up to 56 rows one coefficient block per row (9.08 / 9.46 against 9.29 / 9.53
  // us at 40 / 48 rows, 9.78 / 9.85 against 10.03 / 9.99 at 49 / 52; at 64 rows
  // it was slower, 11.11 against 10.84)
  if (p.do_coeff && p.R <= 56) p.tail_coeff_blocks = p.R;
  const int lcap = 2 * sm_count() - p.tail_coeff_blocks;
  p.tail_layer_blocks = p.do_layer ? (lb < lcap ? lb : lcap) : 0;
  // Up to 4 rows the layer-input blocks are few (7 at 2 rows) and the swizzled
  // scale buffer's padding (127 rows of zeros at 1 row) falls on them: 32 blocks
  // share it (us per boundary, 32 / as many as the tasks need: 5.81 / 6.33 at 1
  // row, 5.73 / 5.91 at 2, 5.81 / 5.89 at 4; at 8 rows it was slower, 6.19 / 5.94).
  if (p.do_layer && p.q_data != nullptr && p.q_swizzled && p.R <= 4 && p.tail_layer_blocks < 32)
    p.tail_layer_blocks = 32 < lcap ? 32 : lcap;
  p.tail_coeff_first = p.R >= kCoeffFirstRows && p.R <= kCoeffFirstMaxRows;
  return launch_pdl(boundary_tail_kernel<N>, p.tail_layer_blocks + p.tail_coeff_blocks, tail_layout<N>().total,
                    stream, p);
}

template <int FRONT>
mhc_status dispatch_n(Params& p, int n, cudaStream_t s) {
  switch (n) {
    case 1: return launch_boundary<1, FRONT>(p, s);
    case 2: return launch_boundary<2, FRONT>(p, s);
    case 4: return launch_boundary<4, FRONT>(p, s);
    default: return MHC_ERR_UNSUPPORTED_SHAPE;
  }
}

// Checks and fills the tail (layer input, MXFP8, coefficients, workspace) shared by
// the two full-boundary entry points.
mhc_status fill_tail(Params& p, const float* pre, const mhc_bf16* norm_weight, float norm_eps,
                     const mhc_coeff_args* coeffs, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
                     float* post_out, float* comb_out, float* pre_out, int R, int H, int n, void* ws,
                     size_t ws_bytes) {
  if (pre == nullptr) {  // residual-only
    if (norm_weight || layer_input || mxfp8 || coeffs) return MHC_ERR_INVALID_ARG;
    p.do_layer = 0;
    p.do_coeff = 0;
    return MHC_OK;
  }
  if (!norm_weight || !layer_input || !aligned(norm_weight, 16) || !aligned(layer_input, 16))
    return MHC_ERR_INVALID_ARG;
  if (!(norm_eps >= 0.f) || !aligned(pre, 4)) return MHC_ERR_INVALID_ARG;
  mhc_status st = check_coeff(coeffs);
  if (st != MHC_OK) return st;
  st = check_mxfp8(mxfp8);
  if (st != MHC_OK) return st;
  if (coeffs && (!post_out || !comb_out || !pre_out)) return MHC_ERR_INVALID_ARG;
  size_t sc2_off, dot_off;
  const size_t need = ws_layout(R, H, n, &sc2_off, &dot_off);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return MHC_ERR_WORKSPACE;
  p.pre = pre;
  p.norm_weight = reinterpret_cast<const __nv_bfloat16*>(norm_weight);
  p.norm_eps = norm_eps;
  p.layer_input = reinterpret_cast<__nv_bfloat16*>(layer_input);
  p.do_layer = 1;
  if (mxfp8) {
    p.q_data = mxfp8->data;
    p.q_scale = mxfp8->scale;
    p.q_swizzled = mxfp8->swizzled_128x4 != 0;
  }
  if (coeffs) {
    p.do_coeff = 1;
    p.fn = coeffs->fn;
    p.fn_packed = static_cast<const __nv_bfloat16*>(coeffs->fn_packed);
    p.scale = coeffs->scale;
    p.base = coeffs->base;
    p.rms_eps = coeffs->rms_eps;
    p.pre_eps = coeffs->pre_eps;
    p.sk_eps = coeffs->sinkhorn_eps;
    p.alpha = coeffs->post_alpha;
    p.iters = coeffs->sinkhorn_iters;
    p.post_out = post_out;
    p.comb_out = comb_out;
    p.pre_out = pre_out;
  }
  p.ctl = static_cast<unsigned*>(ws);
  p.sc2_part = reinterpret_cast<float*>(static_cast<char*>(ws) + sc2_off);
  p.dot_part = reinterpret_cast<float*>(static_cast<char*>(ws) + dot_off);
  return MHC_OK;
}

mhc_status check_mixes(const mhc_bf16* residual, const float* post, const float* comb, mhc_bf16* residual_out) {
  if (!residual || !post || !comb || !residual_out) return MHC_ERR_INVALID_ARG;
  if (!aligned(residual, 16) || !aligned(residual_out, 16) || !aligned(post, 4) || !aligned(comb, 4))
    return MHC_ERR_INVALID_ARG;
  return MHC_OK;
}

}  // namespace

extern "C" {

size_t mhc_workspace_bytes(int rows, int hidden, int hc_mult) {
  if (!shape_ok(rows, hidden, hc_mult)) return 0;
  return ws_layout(rows, hidden, hc_mult, nullptr, nullptr);
}

size_t mhc_mxfp8_scale_bytes(int rows, int hidden, int swizzled_128x4) {
  if (rows < 0 || hidden <= 0 || hidden % 32 != 0) return 0;
  const size_t sc = static_cast<size_t>(hidden / 32);
  if (!swizzled_128x4) return static_cast<size_t>(rows) * sc;
  return static_cast<size_t>((rows + 127) / 128 * 128) * ((sc + 3) / 4 * 4);
}

mhc_status mhc_workspace_init(void* workspace, size_t ws_bytes, mhc_stream stream) {
  if (!workspace || !aligned(workspace, 256) || ws_bytes < kWsHeader) return MHC_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, ws_bytes, stream) != cudaSuccess) return MHC_ERR_CUDA;
  return MHC_OK;
}

}  // extern "C"

namespace {

// mhc_boundary_post_pre over a table of partial pointers (checked by the callers).
mhc_status post_pre_impl(const __nv_bfloat16* const* pptr, int num_partials, bool remote, const mhc_bf16* residual,
                         const float* post, const float* comb, const float* pre, const mhc_bf16* norm_weight,
                         float norm_eps, const mhc_coeff_args* coeffs, mhc_bf16* residual_out, mhc_bf16* aux_out,
                         mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8, float* post_out, float* comb_out,
                         float* pre_out, int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes,
                         mhc_stream stream, bool mailbox = false) {
  mhc_status st = check_mixes(residual, post, comb, residual_out);
  if (st != MHC_OK) return st;
  Params p{};
  for (int u = 0; u < num_partials; ++u) p.pptr[u] = pptr[u];
  p.premote = remote ? 1 : 0;
  p.P = num_partials;
  p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  p.post = post;
  p.comb = comb;
  p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
  p.write_res = 1;
  if (aux_out && !aligned(aux_out, 16)) return MHC_ERR_INVALID_ARG;
  p.aux_out = reinterpret_cast<__nv_bfloat16*>(aux_out);
  p.R = rows;
  p.H = hidden;
  st = fill_tail(p, pre, norm_weight, norm_eps, coeffs, layer_input, mxfp8, post_out, comb_out, pre_out, rows,
                 hidden, hc_mult, workspace, ws_bytes);
  if (st != MHC_OK) return st;
  if (mailbox && p.ctl == nullptr) {  // the slot wait reports through the workspace header
    if (!workspace || !aligned(workspace, 256) || ws_bytes < kWsHeader) return MHC_ERR_WORKSPACE;
    p.ctl = static_cast<unsigned*>(workspace);
  }
  return mailbox ? dispatch_n<kMailbox>(p, hc_mult, stream) : dispatch_n<kPartials>(p, hc_mult, stream);
}

}  // namespace

extern "C" {

mhc_status mhc_boundary_post_pre(const mhc_bf16* partials, int num_partials, int64_t partial_stride,
                                 const mhc_bf16* residual, const float* post, const float* comb, const float* pre,
                                 const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
                                 mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input,
                                 const mhc_mxfp8_out* mxfp8, float* post_out, float* comb_out, float* pre_out,
                                 int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes,
                                 mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (num_partials < 1 || num_partials > kMaxPartials) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!partials || !aligned(partials, 16) || partial_stride % 8 != 0) return MHC_ERR_INVALID_ARG;
  if (num_partials > 1 && partial_stride == 0) return MHC_ERR_INVALID_ARG;
  const __nv_bfloat16* pptr[kMaxPartials];
  for (int u = 0; u < num_partials; ++u)
    pptr[u] = reinterpret_cast<const __nv_bfloat16*>(partials) + static_cast<int64_t>(u) * partial_stride;
  return post_pre_impl(pptr, num_partials, false, residual, post, comb, pre, norm_weight, norm_eps, coeffs,
                       residual_out, aux_out, layer_input, mxfp8, post_out, comb_out, pre_out, rows, hidden, hc_mult,
                       workspace, ws_bytes, stream);
}

mhc_status mhc_boundary_post_pre_ptrs(const mhc_bf16* const* partials, int num_partials, const mhc_bf16* residual,
                                      const float* post, const float* comb, const float* pre,
                                      const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
                                      mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input,
                                      const mhc_mxfp8_out* mxfp8, float* post_out, float* comb_out,
                                      float* pre_out, int rows, int hidden, int hc_mult, void* workspace,
                                      size_t ws_bytes, mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (num_partials < 1 || num_partials > kMaxPartials) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!partials) return MHC_ERR_INVALID_ARG;
  const __nv_bfloat16* pptr[kMaxPartials];
  for (int u = 0; u < num_partials; ++u) {
    if (!partials[u] || !aligned(partials[u], 16)) return MHC_ERR_INVALID_ARG;
    pptr[u] = reinterpret_cast<const __nv_bfloat16*>(partials[u]);
  }
  return post_pre_impl(pptr, num_partials, true, residual, post, comb, pre, norm_weight, norm_eps, coeffs,
                       residual_out, aux_out, layer_input, mxfp8, post_out, comb_out, pre_out, rows, hidden, hc_mult,
                       workspace, ws_bytes, stream);
}

size_t mhc_mailbox_bytes(int world, int max_rows, int hidden) {
  if (world < 1 || world > kMaxPartials || !shape_ok(max_rows, hidden, 1)) return 0;
  return mailbox_total(world, max_rows, hidden);
}

mhc_status mhc_mailbox_init(void* mailbox, size_t bytes, mhc_stream stream) {
  if (!mailbox || !aligned(mailbox, 256) || bytes < kMailboxHeader || bytes % 16 != 0) return MHC_ERR_INVALID_ARG;
  const size_t units = (bytes - kMailboxHeader) / 16;
  const int sms = sm_count();
  size_t blocks = (units + 255) / 256;
  const size_t cap = static_cast<size_t>(sms > 0 ? sms : 1) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  mailbox_init_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<unsigned char*>(mailbox),
                                                                         units);
  if (cudaGetLastError() != cudaSuccess) return MHC_ERR_CUDA;
  return MHC_OK;
}

mhc_status mhc_mailbox_publish(const mhc_bf16* x, int rows, int hidden, int rank, uint32_t round,
                               void* const* mailboxes, int world, int max_rows, mhc_stream stream) {
  if (world < 1 || world > kMaxPartials || !shape_ok(max_rows, hidden, 1) || rows < 1 || rows > max_rows)
    return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!x || !aligned(x, 16) || !mailboxes || rank < 0 || rank >= world || round == 0xffffffffu)
    return MHC_ERR_INVALID_ARG;
  PublishParams q{};
  for (int c = 0; c < world; ++c) {
    if (!mailboxes[c] || !aligned(mailboxes[c], 256)) return MHC_ERR_INVALID_ARG;
    q.mb[c] = static_cast<unsigned char*>(mailboxes[c]);
  }
  q.x = reinterpret_cast<const __nv_bfloat16*>(x);
  q.status = static_cast<unsigned*>(mailboxes[rank]);
  q.rank = rank;
  q.W = world;
  q.M = max_rows;
  q.H = hidden;
  q.round = round;
  q.budget_ns = g_budget_ns;
  mailbox_publish_kernel<<<dim3(rows, world), 256, 0, stream>>>(q);
  if (cudaGetLastError() != cudaSuccess) return MHC_ERR_CUDA;
  return MHC_OK;
}

mhc_status mhc_boundary_collect(void* mailbox, int world, int max_rows, uint32_t round, const mhc_bf16* residual,
                                const float* post, const float* comb, const float* pre,
                                const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
                                mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input,
                                const mhc_mxfp8_out* mxfp8, float* post_out, float* comb_out, float* pre_out,
                                int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes,
                                mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (world < 1 || world > kMaxPartials || max_rows < rows || max_rows > kMaxRows) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!mailbox || !aligned(mailbox, 256) || round == 0xffffffffu) return MHC_ERR_INVALID_ARG;
  const unsigned par = round & 1u;
  unsigned char* mb = static_cast<unsigned char*>(mailbox);
  const __nv_bfloat16* slots = reinterpret_cast<const __nv_bfloat16*>(mb + kMailboxHeader);
  const __nv_bfloat16* pptr[kMaxPartials];
  for (int u = 0; u < world; ++u)
    pptr[u] = slots + (static_cast<size_t>(par) * world + u) * max_rows * static_cast<size_t>(hidden);
  mhc_status st = post_pre_impl(pptr, world, true, residual, post, comb, pre, norm_weight, norm_eps, coeffs,
                                residual_out, aux_out, layer_input, mxfp8, post_out, comb_out, pre_out, rows, hidden,
                                hc_mult, workspace, ws_bytes, stream, true);
  if (st != MHC_OK) return st;
  // an ordinary launch: it runs once the boundary has read (and re-marked) every
  // slot of this round, and leaves the round unconsumed if the boundary recorded
  // an error (a slot wait that ran out), so that producers report it too
  mailbox_done_kernel<<<1, 1, 0, stream>>>(reinterpret_cast<unsigned*>(mb + 8), par, round + 1u,
                                           static_cast<const unsigned*>(workspace));
  if (cudaGetLastError() != cudaSuccess) return MHC_ERR_CUDA;
  return MHC_OK;
}

mhc_status mhc_boundary_moe_finalize(const mhc_bf16* gemm2_permuted, int num_permuted, const float* expert_weights,
                                     const int32_t* expanded_idx_to_permuted_idx, int top_k,
                                     const mhc_bf16* shared_output, const mhc_bf16* residual, const float* post,
                                     const float* comb, const float* pre, const mhc_bf16* norm_weight,
                                     float norm_eps, const mhc_coeff_args* coeffs, mhc_bf16* residual_out,
                                     mhc_bf16* aux_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
                                     float* post_out,
                                     float* comb_out, float* pre_out, int rows, int hidden, int hc_mult,
                                     void* workspace, size_t ws_bytes, mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (top_k < 1 || top_k > kMaxTopK || num_permuted < 0) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!gemm2_permuted || !expert_weights || !expanded_idx_to_permuted_idx || !shared_output)
    return MHC_ERR_INVALID_ARG;
  if (!aligned(gemm2_permuted, 16) || !aligned(shared_output, 16) || !aligned(expert_weights, 4) ||
      !aligned(expanded_idx_to_permuted_idx, 4))
    return MHC_ERR_INVALID_ARG;
  mhc_status st = check_mixes(residual, post, comb, residual_out);
  if (st != MHC_OK) return st;
  Params p{};
  p.gemm2 = reinterpret_cast<const __nv_bfloat16*>(gemm2_permuted);
  p.num_perm = num_permuted;
  p.ew = expert_weights;
  p.e2p = expanded_idx_to_permuted_idx;
  p.topk = top_k;
  p.shared_out = reinterpret_cast<const __nv_bfloat16*>(shared_output);
  p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  p.post = post;
  p.comb = comb;
  p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
  p.write_res = 1;
  if (aux_out && !aligned(aux_out, 16)) return MHC_ERR_INVALID_ARG;
  p.aux_out = reinterpret_cast<__nv_bfloat16*>(aux_out);
  p.R = rows;
  p.H = hidden;
  // the MoE routing of every row is staged in shared memory; the residual-only
  // form still needs the workspace header for the status word
  st = fill_tail(p, pre, norm_weight, norm_eps, coeffs, layer_input, mxfp8, post_out, comb_out, pre_out, rows,
                 hidden, hc_mult, workspace, ws_bytes);
  if (st != MHC_OK) return st;
  if (pre == nullptr) {
    if (!workspace || !aligned(workspace, 256) || ws_bytes < kWsHeader) return MHC_ERR_WORKSPACE;
    p.ctl = static_cast<unsigned*>(workspace);
  }
  return dispatch_n<kMoe>(p, hc_mult, stream);
}

mhc_status mhc_boundary_residual_only(const mhc_bf16* partials, int num_partials, int64_t partial_stride,
                                      const mhc_bf16* residual, const float* post, const float* comb,
                                      mhc_bf16* residual_out, mhc_bf16* aux_out, int rows, int hidden,
                                      int hc_mult, mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (num_partials < 1 || num_partials > kMaxPartials) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!partials || !aligned(partials, 16) || partial_stride % 8 != 0) return MHC_ERR_INVALID_ARG;
  if (num_partials > 1 && partial_stride == 0) return MHC_ERR_INVALID_ARG;
  mhc_status st = check_mixes(residual, post, comb, residual_out);
  if (st != MHC_OK) return st;
  Params p{};
  for (int u = 0; u < num_partials; ++u)
    p.pptr[u] = reinterpret_cast<const __nv_bfloat16*>(partials) + static_cast<int64_t>(u) * partial_stride;
  p.P = num_partials;
  p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  p.post = post;
  p.comb = comb;
  p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
  p.write_res = 1;
  if (aux_out && !aligned(aux_out, 16)) return MHC_ERR_INVALID_ARG;
  p.aux_out = reinterpret_cast<__nv_bfloat16*>(aux_out);
  p.R = rows;
  p.H = hidden;
  return dispatch_n<kPartials>(p, hc_mult, stream);
}

mhc_status mhc_coeffs(const mhc_bf16* residual, const mhc_coeff_args* coeffs, const float* pre_mix,
                      const mhc_bf16* x, mhc_bf16* residual_out, const mhc_bf16* norm_weight, float norm_eps,
                      mhc_bf16* layer_input, float* post_out, float* comb_out, float* pre_out, int rows,
                      int hidden, int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if ((residual == nullptr) == (x == nullptr)) return MHC_ERR_INVALID_ARG;
  if (!coeffs || !post_out || !comb_out || !pre_out) return MHC_ERR_INVALID_ARG;
  mhc_status st = check_coeff(coeffs);
  if (st != MHC_OK) return st;
  size_t sc2_off, dot_off;
  const size_t need = ws_layout(rows, hidden, hc_mult, &sc2_off, &dot_off);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < need) return MHC_ERR_WORKSPACE;
  Params p{};
  p.R = rows;
  p.H = hidden;
  p.do_coeff = 1;
  p.fn = coeffs->fn;
  p.fn_packed = static_cast<const __nv_bfloat16*>(coeffs->fn_packed);
  p.scale = coeffs->scale;
  p.base = coeffs->base;
  p.rms_eps = coeffs->rms_eps;
  p.pre_eps = coeffs->pre_eps;
  p.sk_eps = coeffs->sinkhorn_eps;
  p.alpha = coeffs->post_alpha;
  p.iters = coeffs->sinkhorn_iters;
  p.post_out = post_out;
  p.comb_out = comb_out;
  p.pre_out = pre_out;
  p.ctl = static_cast<unsigned*>(workspace);
  p.sc2_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + sc2_off);
  p.dot_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + dot_off);
  if (layer_input) {
    if (!norm_weight || !aligned(norm_weight, 16) || !aligned(layer_input, 16) || !(norm_eps >= 0.f))
      return MHC_ERR_INVALID_ARG;
    p.do_layer = 1;
    p.norm_weight = reinterpret_cast<const __nv_bfloat16*>(norm_weight);
    p.norm_eps = norm_eps;
    p.layer_input = reinterpret_cast<__nv_bfloat16*>(layer_input);
  }
  if (x) {
    if (pre_mix || !aligned(x, 16)) return MHC_ERR_INVALID_ARG;
    if (residual_out && !aligned(residual_out, 16)) return MHC_ERR_INVALID_ARG;
    p.x = reinterpret_cast<const __nv_bfloat16*>(x);
    p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
    p.write_res = residual_out != nullptr;
    return dispatch_n<kBroadcast>(p, hc_mult, stream);
  }
  if (residual_out || !aligned(residual, 16)) return MHC_ERR_INVALID_ARG;
  if (layer_input && (!pre_mix || !aligned(pre_mix, 4))) return MHC_ERR_INVALID_ARG;
  p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  p.pre = pre_mix;
  return dispatch_n<kStreams>(p, hc_mult, stream);
}

mhc_status mxfp8_quantize_rows(const mhc_bf16* x, int rows, int hidden, const mhc_mxfp8_out* out,
                               mhc_stream stream) {
  if (rows < 1 || rows > 65535 || hidden < 32 || hidden % 32 != 0) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!x || !aligned(x, 16) || check_mxfp8(out) != MHC_OK || out == nullptr) return MHC_ERR_INVALID_ARG;
  const long long lanes = static_cast<long long>(rows) * (hidden / 8);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((lanes + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, mxfp8_rows_kernel, reinterpret_cast<const __nv_bfloat16*>(x), rows, hidden, out->data,
                         out->scale, static_cast<int>(out->swizzled_128x4 != 0)) != cudaSuccess) {
    (void)cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  if (out->swizzled_128x4) {
    const int scols = hidden / 32;
    const int rows_p = (rows + 127) / 128 * 128;
    const int cols_p = (scols + 3) / 4 * 4;
    if (rows_p != rows || cols_p != scols) {
      const int total = rows_p * cols_p;
      cfg.gridDim = dim3((total + 255) / 256 < 1024 ? (total + 255) / 256 : 1024);
      if (cudaLaunchKernelEx(&cfg, scale_padding_kernel, out->scale, rows, hidden) != cudaSuccess) {
        (void)cudaGetLastError();
        return MHC_ERR_CUDA;
      }
    }
  }
  return MHC_OK;
}

size_t mhc_projection_pack_bytes(int hidden, int hc_mult) {
  if (!shape_ok(1, hidden, hc_mult)) return 0;
  const int G = hidden / kCols;
  const int pb = hc_mult == 1 ? packed_slice_bytes(1) : (hc_mult == 2 ? packed_slice_bytes(2) : packed_slice_bytes(4));
  return static_cast<size_t>(G) * pb;
}

mhc_status mhc_projection_pack(const float* fn, void* packed, int hidden, int hc_mult, mhc_stream stream) {
  if (!shape_ok(1, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!fn || !packed || !aligned(fn, 4) || !aligned(packed, 16)) return MHC_ERR_INVALID_ARG;
  const int G = hidden / kCols;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(packed);
  switch (hc_mult) {
    case 1: pack_projection_kernel<1><<<G, 256, 0, stream>>>(fn, hidden, out); break;
    case 2: pack_projection_kernel<2><<<G, 256, 0, stream>>>(fn, hidden, out); break;
    default: pack_projection_kernel<4><<<G, 256, 0, stream>>>(fn, hidden, out); break;
  }
  if (cudaGetLastError() != cudaSuccess) return MHC_ERR_CUDA;
  return MHC_OK;
}

}  // extern "C"

namespace {

// Exported handle: the CUDA IPC handle of the allocation that holds the
// pointer, then the pointer's byte offset into it.
struct IpcHandle {
  cudaIpcMemHandle_t mem;
  uint64_t offset;
};

// Base of the allocation holding p (the IPC handle covers a whole allocation),
// through the driver's cuMemGetAddressRange, looked up once.
bool allocation_base(const void* p, uintptr_t* base) {
  typedef int (*GetRange)(uintptr_t*, size_t*, uintptr_t);
  static GetRange fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetRange>(f);
  });
  if (fn == nullptr) return false;
  size_t size = 0;
  return fn(base, &size, reinterpret_cast<uintptr_t>(p)) == 0;
}

std::mutex g_ipc_mu;
std::map<uintptr_t, uintptr_t> g_ipc_open;  // pointer handed out -> mapped base

}  // namespace

extern "C" {

size_t mhc_ipc_handle_bytes(void) { return sizeof(IpcHandle); }

mhc_status mhc_ipc_export(const void* dev_ptr, void* handle_out) {
  if (!dev_ptr || !handle_out) return MHC_ERR_INVALID_ARG;
  uintptr_t base = 0;
  if (!allocation_base(dev_ptr, &base)) return MHC_ERR_CUDA;
  IpcHandle h{};
  if (cudaIpcGetMemHandle(&h.mem, reinterpret_cast<void*>(base)) != cudaSuccess) {
    (void)cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  h.offset = reinterpret_cast<uintptr_t>(dev_ptr) - base;
  std::memcpy(handle_out, &h, sizeof(h));
  return MHC_OK;
}

mhc_status mhc_ipc_import(const void* handle, void** dev_ptr_out) {
  if (!handle || !dev_ptr_out) return MHC_ERR_INVALID_ARG;
  IpcHandle h;
  std::memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h.mem, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    (void)cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  const uintptr_t ptr = reinterpret_cast<uintptr_t>(base) + h.offset;
  {
    std::lock_guard<std::mutex> lock(g_ipc_mu);
    g_ipc_open[ptr] = reinterpret_cast<uintptr_t>(base);
  }
  *dev_ptr_out = reinterpret_cast<void*>(ptr);
  return MHC_OK;
}

mhc_status mhc_ipc_release(void* dev_ptr) {
  uintptr_t base = 0;
  {
    std::lock_guard<std::mutex> lock(g_ipc_mu);
    auto it = g_ipc_open.find(reinterpret_cast<uintptr_t>(dev_ptr));
    if (it == g_ipc_open.end()) return MHC_ERR_INVALID_ARG;
    base = it->second;
    g_ipc_open.erase(it);
  }
  if (cudaIpcCloseMemHandle(reinterpret_cast<void*>(base)) != cudaSuccess) {
    (void)cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  return MHC_OK;
}

mhc_status mhc_get_device_status(void* workspace, mhc_stream stream) {
  if (!workspace || !aligned(workspace, 256)) return MHC_ERR_WORKSPACE;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MHC_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MHC_ERR_CUDA;
  if (v != 0 && cudaMemset(workspace, 0, sizeof(v)) != cudaSuccess) return MHC_ERR_CUDA;
  return static_cast<mhc_status>(v);
}

const char* mhc_status_string(mhc_status s) {
  switch (s) {
    case MHC_OK: return "MHC_OK";
    case MHC_ERR_INVALID_ARG: return "MHC_ERR_INVALID_ARG";
    case MHC_ERR_UNSUPPORTED_SHAPE: return "MHC_ERR_UNSUPPORTED_SHAPE";
    case MHC_ERR_WORKSPACE: return "MHC_ERR_WORKSPACE";
    case MHC_ERR_CUDA: return "MHC_ERR_CUDA";
    case MHC_ERR_DEVICE_TIMEOUT: return "MHC_ERR_DEVICE_TIMEOUT";
    case MHC_ERR_DEVICE_INDEX: return "MHC_ERR_DEVICE_INDEX";
  }
  return "MHC_ERR_UNKNOWN";
}

int64_t mhc_debug_set_wait(int64_t budget_ns, int extra_units) {
  const int64_t old = g_budget_ns;
  if (budget_ns > 0) g_budget_ns = budget_ns;
  g_extra_tx = extra_units < 0 ? 0 : extra_units;
  return old;
}

// ---------------------------------------------------------------------------
// Boundary without a caller-provided workspace.
//
// Some callers cannot allocate device memory: a plugin hosted by a runtime
// that owns all device memory and only hands it tensors, code that runs while
// a CUDA graph is being captured (cudaMalloc is not a stream operation), or a
// serving loop that must never take the allocator's locks. For them the
// scratch of mhc_boundary_post_pre lives in the fixed array below, which every
// GPU that loads the library holds until the process exits.

}  // extern "C"

namespace {

constexpr int kNoAllocMaxRows = 128;
constexpr int kNoAllocMaxHidden = 7168;
constexpr int kNoAllocMaxHc = 4;
// mhc_workspace_bytes(128, 7168, 4): header, c^2 sums [128][112] (rounded to
// 256 bytes), projection sums [128][112][32] floats
constexpr size_t kNoAllocBytes = kWsHeader + ((static_cast<size_t>(kNoAllocMaxRows) * (kNoAllocMaxHidden / kCols) * 4 + 255) & ~static_cast<size_t>(255)) +
                                 static_cast<size_t>(kNoAllocMaxRows) * (kNoAllocMaxHidden / kCols) * red_of(kNoAllocMaxHc) * 4;

// The array is zero at module load. A kernel never needs its contents to start
// at zero except the status word, which only a failed wait writes.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// The calling thread's current CUDA context (the driver's cuCtxGetCurrent), or
// null where the driver entry point is unavailable.
void* current_context() {
  typedef int (*CtxGetCurrent)(void**);
  static CtxGetCurrent fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrent>(f);
    else
      (void)cudaGetLastError();
  });
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the array on the current device. In host code the symbol is
// only a host-side stand-in; the kernels get this address. It is looked up once
// per device and context: a device reset gives the device a new primary context,
// in which the module is loaded again, so the address is looked up again.
void* noalloc_scratch() {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  static void* ctx_of[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] != nullptr && ctx_of[dev] != nullptr && current_context() == ctx_of[dev]) return addr[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {  // also makes the context current
    (void)cudaGetLastError();
    return nullptr;
  }
  addr[dev] = p;
  ctx_of[dev] = current_context();
  return p;
}

}  // namespace

extern "C" {

mhc_status mhc_boundary_post_pre_noalloc(const mhc_bf16* partials, int num_partials, int64_t partial_stride,
                                         const mhc_bf16* residual, const float* post, const float* comb,
                                         const float* pre, const mhc_bf16* norm_weight, float norm_eps,
                                         const mhc_coeff_args* coeffs, mhc_bf16* residual_out,
                                         mhc_bf16* aux_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
                                         float* post_out, float* comb_out, float* pre_out, int rows, int hidden,
                                         int hc_mult, mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (rows > kNoAllocMaxRows || hidden > kNoAllocMaxHidden || hc_mult > kNoAllocMaxHc ||
      ws_layout(rows, hidden, hc_mult, nullptr, nullptr) > kNoAllocBytes)
    return MHC_ERR_WORKSPACE;  // needs more scratch than the fixed array holds
  void* ws = noalloc_scratch();
  if (ws == nullptr) return MHC_ERR_CUDA;
  return mhc_boundary_post_pre(partials, num_partials, partial_stride, residual, post, comb, pre, norm_weight,
                               norm_eps, coeffs, residual_out, aux_out, layer_input, mxfp8, post_out, comb_out,
                               pre_out, rows, hidden, hc_mult, ws, kNoAllocBytes, stream);
}

}  // extern "C"
