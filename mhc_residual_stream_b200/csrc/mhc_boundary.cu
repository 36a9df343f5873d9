// mHC decode boundary on B200 (sm_100a): the fused kernel and the C ABI of
// libmhc.so (declared in include/mhc.h).
//
// A boundary is ONE launch of boundary_kernel over G = H/64 CTAs, one per SM.
// CTA g owns columns [64g, 64g + 64) of every row, so every weight of fn is
// read from HBM exactly once per boundary.
//   1. Before it waits for its predecessor on the stream (programmatic dependent
//      launch), a CTA starts the bulk copy of its fn slice (fp32) into shared
//      memory.
//   2. After the wait, tensor-map TMA loads bring the rows' data into shared
//      memory in 16-row chunks, up to four in flight: the partials (one 3-D
//      box), or the MoE expert rows gathered by index (tile::gather4) and the
//      shared output, and the residual streams (one 3-D box). While they are in
//      flight the CTA splits each fn weight into three bf16 terms (128B-swizzled
//      rows of K values, one row per term and fn column).
//   3. Two groups of eight warps take alternate chunks: sum or finalize x, mHC
//      post-mix (vllm ...boundary.boundary, Boundaries.post_only: mhc_post(x,
//      residual, post, comb)), store the new streams, stage them in shared
//      memory, and sum per row the squares of their collapse with the carried
//      pre (BoundaryState.pre) and of the streams.
//   4. The same warps project the chunk's 16 rows of staged streams onto the C
//      fn columns on the tensor cores (mma.sync m16n8k16 bf16, fp32
//      accumulation; each warp a share of K, the shares added in warp order),
//      while a control warp refills the chunk's stage.
//   5. Each CTA publishes its row records (C dot products, sum v^2, sum c^2) as
//      tagged 64-bit words in the workspace, field-major, so that one field of
//      one row is contiguous over the CTAs (no flag, no fence, no second kernel).
//   6. In one round over the published words every CTA adds the sum of c^2 of
//      every row and the records of the rows whose coefficients it finishes
//      (rows g and g + G), writes its columns of the layer input (and MXFP8),
//      and runs those rows' logits, sigmoid and Sinkhorn.
// The residual-only variant is steps 2-3 alone. Every reduction runs in a fixed
// order, so results are bitwise reproducible.

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

constexpr int kCols = 64;        // columns of H per CTA
constexpr int kRC = 16;          // rows per chunk (N of one projection MMA)
constexpr int kMaxStages = 4;    // chunks in flight (fewer where they do not fit in shared memory)
constexpr int kWorkWarps = 16;   // warps of the streaming phase: two groups of 8 on alternate chunks
constexpr int kGroupWarps = 8;   // a group: 2 rows of a chunk per warp, 4 columns per lane
constexpr int kCtl = kWorkWarps; // index of the control warp
constexpr int kThreads = (kWorkWarps + 1) * 32;
constexpr int kWorkThreads = kWorkWarps * 32;
constexpr int kMaxRows = 128;
constexpr int kMaxChunks = kMaxRows / kRC;
constexpr int kMaxPartials = 16;
constexpr int kMaxTopK = 16;
constexpr int kMaxIters = 1000;
constexpr int kMaxBlocks = 148;
constexpr int kRecF = 32;        // shared-memory stride of a row record: C dot products, sum v^2, sum c^2
// Workspace: a 1 KB header (status word at byte 0, the launch epoch at byte 64),
// then the CTAs' row records as tagged 64-bit words, [G CTAs][R rows][fields],
// then the rows' total sums of c^2, one copy for each CTA to read, [G][R].
constexpr size_t kWsHeader = 1024;
constexpr int kStatusWord = 0;
constexpr int kEpochWord = 16;

enum Front { kPartials = 0, kMoe = 1, kStreams = 2, kBroadcast = 3, kMailbox = 4, kTable = 5 };
// Fronts whose x is a sum of P bf16 partials read by the lanes themselves (a table
// of pointers that may be other GPUs' memory, or the slots of a mailbox that
// producers fill concurrently, each element valid once it is not negative zero).
__host__ __device__ constexpr bool lane_partials(int front) { return front == kMailbox || front == kTable; }

__host__ __device__ constexpr int logits_of(int n) { return 2 * n + n * n; }
// Fields of a published row record: C dot products, sum v^2 and sum c^2, rounded
// up to an even count (records are read as 16-byte pairs of words).
__host__ __device__ constexpr int fields_of(int n) { return (logits_of(n) + 3) & ~1; }
// rows of the fn slice image: three bf16 terms of each of the C fn columns (row
// t*C + c), rounded up to a whole 8-row swizzle atom
__host__ __device__ constexpr int arows_of(int n) { return (3 * logits_of(n) + 7) & ~7; }
// Bytes of a CTA's fn slice image (mhc_projection_pack).
__host__ __device__ constexpr int aimage_bytes(int n) { return n * arows_of(n) * 128; }

struct Params {
  // front ends
  const __nv_bfloat16* pptr[kMaxPartials];  // lane-read partials: [R, H] at pptr[u]
  int P;
  int premote;  // partials may be other GPUs' memory (L2-only loads)
  const __nv_bfloat16* gemm2;
  int num_perm;
  const float* ew;
  const int32_t* e2p;
  int topk;
  const float* post;
  const float* comb;
  const float* pre;  // carried pre (boundary) or pre_mix (coefficients entry)
  // layer input
  const __nv_bfloat16* norm_weight;
  float norm_eps;
  // coefficients
  const float* fn;
  const unsigned char* fn_packed;  // [G] A operand images, or null
  const float* scale;
  const float* base;
  float rms_eps, pre_eps, sk_eps, alpha;
  int iters;
  // outputs
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
  int stages;  // chunk stages in flight: 1 .. kMaxStages
  // workspace
  unsigned* ctl;             // header: status, epoch
  unsigned long long* rec;   // [G][R][fields] tagged words: the CTAs' row records
  unsigned long long* tot;   // [G][R] tagged words: the rows' sums c^2, one copy per CTA
  int extra_tx;  // test hook: 16-byte units the fn wait expects beyond what arrives
  int64_t budget_ns;
};

// Shared memory of the kernel, offsets from a 1024-byte aligned base.
struct Layout {
  int a_off, v_off, st_off, stage_bytes, res_units, fst_off, part_off, mix_off, moe_off, rec_off, inv_off, cft_off,
      bar_off, total;
  int r_alloc;
};

// Bytes of one chunk's projection partials: [warp][16 rows][C] floats.
__host__ __device__ constexpr int part_bytes(int n) { return kGroupWarps * kRC * logits_of(n) * 4; }

// 128-byte box rows of one chunk's stage, and where the residual streams start.
__host__ __device__ inline void stage_units(int front, int n, int P, int topk, int* units, int* res_units) {
  int u = 0, ru = 0;
  switch (front) {
    case kPartials: ru = P * kRC; u = ru + n * kRC; break;
    case kMoe: ru = (topk + 1) * kRC; u = ru + n * kRC; break;
    case kBroadcast: ru = 0; u = kRC; break;
    default: ru = 0; u = n * kRC; break;  // streams, table, mailbox: the residual streams only
  }
  *units = u;
  *res_units = ru;
}

template <int N>
__host__ __device__ inline Layout layout_of(int front, int R, int G, int P, int topk, bool coeff, bool layer,
                                          int stages, bool packed) {
  constexpr int C = logits_of(N);
  Layout L{};
  L.r_alloc = (R + kRC - 1) / kRC * kRC;
  int o = 0;
  L.a_off = o;  // fn slice image [n atom columns][arows][128 B]
  if (coeff) o += aimage_bytes(N);
  // new streams [n atom columns][r_alloc][128 B]; until the first chunk is
  // staged, the fp32 fn slice as copied, [n][64][C]
  L.v_off = L.fst_off = o;
  int vb = (coeff || layer) ? N * L.r_alloc * 128 : 0;
  if (coeff && !packed && vb < N * kCols * C * 4) vb = N * kCols * C * 4;
  o += vb;
  L.st_off = o;  // chunk stages
  int units, ru;
  stage_units(front, N, P, topk, &units, &ru);
  L.stage_bytes = units * 128;
  L.res_units = ru;
  // after the last chunk, the row records this CTA adds up: [ceil(R / G) * G][fields]
  int st = stages * L.stage_bytes;
  if ((coeff || layer) && st < (R + G - 1) / G * G * fields_of(N) * 4) st = (R + G - 1) / G * G * fields_of(N) * 4;
  o += st;
  // a chunk's projection partials go into its consumed stage when they fit
  // (the stage is refilled only once the chunk is done), else here, one
  // buffer per group
  L.part_off = -1;
  if (coeff && L.stage_bytes < part_bytes(N)) {
    L.part_off = o;
    o += 2 * part_bytes(N);
  }
  L.mix_off = o;  // [R][post n | comb n*n | pre n]
  o += (R * (2 * N + N * N) * 4 + 15) & ~15;
  L.moe_off = o;  // e2p [R*topk], weights [R*topk]
  if (front == kMoe) o += (R * topk * 8 + 15) & ~15;
  L.rec_off = o;  // this CTA's row records [R][kRecF]
  if (coeff || layer) o += R * kRecF * 4;
  L.inv_off = o;  // [R] inverse RMS of the collapse
  if (layer) o += (R * 4 + 15) & ~15;
  L.cft_off = o;  // [ceil(R / G)][kRecF] the totals of the rows this CTA adds up
  if (coeff || layer) o += (R + G - 1) / G * kRecF * 4;
  L.bar_off = o;  // full[kMaxStages], vready[kMaxChunks], fnbar, then the tag slot
  o += (kMaxStages + kMaxChunks + 1) * 8 + 16;
  L.total = (o + 15) & ~15;
  return L;
}


__device__ __forceinline__ int swizzled_scale_offset(int r, int c, int col_tiles) {
  const int tile = (r >> 7) * col_tiles + (c >> 2);
  const int rr = r & 127;
  return tile * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3);
}

// Byte offset of (row, 4-column group v of 16) in a 128B-swizzled K-major atom
// column: rows of 128 bytes, 16-byte chunk index XOR-ed with row % 8.
__device__ __forceinline__ int sw128_offset(int row, int v) {
  return row * 128 + ((((v >> 1) ^ row) & 7) << 4) + (v & 1) * 8;
}

__device__ __forceinline__ uint2 lds_v2(const void* p) { return *reinterpret_cast<const uint2*>(p); }

__device__ __forceinline__ void named_sync_workers() {  // the streaming warps (groups use barriers 1 and 2)
  asm volatile("bar.sync 3, %0;" ::"n"(kWorkThreads) : "memory");
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

// Eight consecutive K values (kin = 8*oct .. 8*oct + 7) of fn column c, read from
// the fp32 slice [kin][C], written as the three terms' 16-byte chunks of A rows
// c, C + c and 2C + c in atom column j.
template <int N>
__device__ __forceinline__ void split_octet(const float* slice, unsigned char* a_col, int c, int oct) {
  constexpr int C = logits_of(N);
  unsigned w[3][4];
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    __nv_bfloat16 h0, m0, l0, h1, m1, l1;
    split3(slice[(oct * 8 + e) * C + c], h0, m0, l0);
    split3(slice[(oct * 8 + e + 1) * C + c], h1, m1, l1);
    w[0][e / 2] = static_cast<unsigned>(__bfloat16_as_ushort(h0)) | (static_cast<unsigned>(__bfloat16_as_ushort(h1)) << 16);
    w[1][e / 2] = static_cast<unsigned>(__bfloat16_as_ushort(m0)) | (static_cast<unsigned>(__bfloat16_as_ushort(m1)) << 16);
    w[2][e / 2] = static_cast<unsigned>(__bfloat16_as_ushort(l0)) | (static_cast<unsigned>(__bfloat16_as_ushort(l1)) << 16);
  }
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    const int m = t * C + c;
    *reinterpret_cast<uint4*>(a_col + m * 128 + (((oct ^ m) & 7) << 4)) = make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
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


// The coefficients of row r, by one warp, from the row's totals over the CTAs
// (tot[c]: dot product with fn column c, tot[C]: sum v^2): the logits (lane c
// computes logit c), pre / post by sigmoid, and the comb by one exponential per
// lane and Sinkhorn in lane 0 ([boundary] Boundaries.sublayer:
// mhc_pre_delayed_overlap(residual, fn, scale, base, rms_norm_eps, hc_eps,
// hc_eps, hc_post_alpha, hc_sinkhorn_iters)).
template <int N>
__device__ __forceinline__ void coefficient_row(const Params& p, int r, const float* tot, float scale_l, float base_l,
                                                int lane) {
  constexpr int C = logits_of(N);
  constexpr int NN = N * N;
  const float s = lane < C ? tot[lane] : 0.f;
  const float inv = rsqrtf(__fdiv_rn(tot[C], static_cast<float>(N * p.H)) + p.rms_eps);
  const float l = lane < C ? scale_l * inv * s + base_l : 0.f;
  if (lane < N) {
    p.pre_out[r * N + lane] = 1.f / (1.f + expf(-l)) + p.pre_eps;
  } else if (lane < 2 * N) {
    p.post_out[r * N + (lane - N)] = p.alpha / (1.f + expf(-l));
  }
  // M = exp(L - max L) with one exp per lane, then Sinkhorn in one thread
  const float lk = __shfl_sync(kFull, l, (lane + 2 * N) & 31);  // lane k < n*n: comb logit k
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

// The projection of chunk c's 16 staged rows (K = n*64 stream values each) onto
// the C fn columns on the tensor cores, by the 8 warps of the chunk's group:
// warp wq runs K steps wq, wq + 8, ... (16 values each: stream k / 4, offset
// 16 * (k % 4)), one accumulator per bf16 term of fn; the terms are added
// (hi + mid) + lo and the warp's 16 x C partial sums go to part[wq].
template <int N>
__device__ __forceinline__ void project_chunk(const unsigned char* f_s, const unsigned char* v_s, int r_alloc, int c,
                                              int wq, int lane, float* part) {
  constexpr int C = logits_of(N);
  constexpr int AR = arows_of(N);
  constexpr int NT = (C + 7) / 8;  // 8-column tiles
  float acc[3][NT][4];
#pragma unroll
  for (int t = 0; t < 3; ++t)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[t][nt][q] = 0.f;
  for (int k = wq; k < 4 * N; k += kGroupWarps) {
    const int j = k >> 2, kc0 = (k & 3) * 2;  // two 16-byte chunks of a 128-byte row
    const int row = c * kRC + (lane & 15), kca = kc0 + (lane >> 4);
    unsigned a[4];
    ldmatrix_x4(a, v_s + j * r_alloc * 128 + row * 128 + (((kca ^ row) & 7) << 4));
    const int kcb = kc0 + ((lane >> 3) & 1);
#pragma unroll
    for (int t = 0; t < 3; ++t) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = t * C + nt * 8 + (lane & 7);  // columns past C read other rows: ignored below
        unsigned b[2];
        ldmatrix_x2(b, f_s + j * AR * 128 + m * 128 + (((kcb ^ m) & 7) << 4));
        mma_bf16_16816(acc[t][nt], a, b);
      }
    }
  }
  // C fragment: lane holds rows lane/4 and lane/4 + 8, columns 2*(lane%4) + {0, 1}
  float* dst = part + wq * kRC * C;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rr = (lane >> 2) + 8 * h;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = nt * 8 + 2 * (lane & 3) + e;
        if (col < C) dst[rr * C + col] = (acc[0][nt][2 * h + e] + acc[1][nt][2 * h + e]) + acc[2][nt][2 * h + e];
      }
    }
  }
}

__device__ __forceinline__ float sum16_lanes(float v) {  // over the 16 lanes sharing lane bit 4
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

__device__ __forceinline__ void named_sync_group(int q) {  // barrier ids are immediates: 1 and 2
  if (q == 0) {
    asm volatile("bar.sync 1, %0;" ::"n"(kGroupWarps * 32) : "memory");
  } else {
    asm volatile("bar.sync 2, %0;" ::"n"(kGroupWarps * 32) : "memory");
  }
}

// The boundary, one launch. See the top of this file for the steps; the
// numbered comments below follow them.
template <int N, int FRONT>
__global__ void __launch_bounds__(kThreads, 1)
    boundary_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_res, const __grid_constant__ CUtensorMap tm_gather) {
  constexpr int C = logits_of(N);
  constexpr int MIX = 2 * N + N * N;
  constexpr int AR = arows_of(N);
  constexpr int NFP = fields_of(N);  // record fields: C dot products, sum v^2, sum c^2 (even)
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  const int R = p.R, H = p.H;
  const int G = gridDim.x;
  const bool coeff = p.do_coeff != 0, layer = p.do_layer != 0, exch = coeff || layer;
  const int S = p.stages;
  const bool packed = p.fn_packed != nullptr;
  const Layout L = layout_of<N>(FRONT, R, G, p.P, p.topk, coeff, layer, S, packed);
  unsigned char* a_s = smem + L.a_off;
  unsigned char* v_s = smem + L.v_off;
  unsigned char* st_s = smem + L.st_off;
  unsigned char* fst_s = smem + L.fst_off;  // the fp32 fn slice as copied
  float* mix_s = reinterpret_cast<float*>(smem + L.mix_off);
  int* e2p_s = reinterpret_cast<int*>(smem + L.moe_off);
  float* ew_s = reinterpret_cast<float*>(smem + L.moe_off) + R * p.topk;
  float* rec_s = reinterpret_cast<float*>(smem + L.rec_off);  // [R][kRecF] this CTA's row records
  float* inv_s = reinterpret_cast<float*>(smem + L.inv_off);  // [R] inverse RMS of the collapse
  float* cft_s = reinterpret_cast<float*>(smem + L.cft_off);  // [slot][kRecF] this CTA's coefficient rows' totals
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* vready = full + kMaxStages;
  uint64_t* fnbar = vready + kMaxChunks;
  uint32_t* tag_slot = reinterpret_cast<uint32_t*>(fnbar + 1);

  const int g = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nch = (R + kRC - 1) / kRC;
  const long long deadline = wait_deadline(p.budget_ns);
  unsigned* status = p.ctl ? p.ctl + kStatusWord : nullptr;  // null: a residual-only call without a workspace
  // the streaming lanes: group q of 8 warps takes chunks q, q + 2, ...; in a
  // chunk, row rl = 2 * (warp % 8) + lane / 16 and columns h0 .. h0 + 3
  const int q = warp / kGroupWarps, wq = warp % kGroupWarps;
  const int rl = wq * 2 + (lane >> 4);
  const int v = lane & 15;
  const int h0 = g * kCols + v * 4;

  // ---- 1. set-up before the wait (no kernel of this library writes weights,
  // and kernels that do not trigger dependent launches are waited for in full
  // before this one starts): the fn slice's copy goes out first
  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    for (int c = 0; c < nch; ++c) mbar_init(&vready[c], kGroupWarps);
    mbar_init(fnbar, 1);
    if (coeff) {
      if (packed) {
        mbar_arrive_expect_tx(fnbar, aimage_bytes(N) + 16 * p.extra_tx);
        bulk_g2s(a_s, p.fn_packed + static_cast<size_t>(g) * aimage_bytes(N), aimage_bytes(N), fnbar);
      } else {
        constexpr int JB = kCols * C * 4;  // one stream's 64 rows of fn: contiguous
        mbar_arrive_expect_tx(fnbar, N * JB + 16 * p.extra_tx);
#pragma unroll
        for (int j = 0; j < N; ++j)
          bulk_g2s(fst_s + j * JB, p.fn + (static_cast<size_t>(j) * H + g * kCols) * C, JB, fnbar);
      }
    }
    if (FRONT == kPartials || FRONT == kBroadcast || FRONT == kMoe) prefetch_tensormap(&tm_x);
    if (FRONT != kBroadcast) prefetch_tensormap(&tm_res);
    if (FRONT == kMoe && p.num_perm > 0) prefetch_tensormap(&tm_gather);
  }
  uint2 nw = make_uint2(0, 0);  // this lane's 4 norm weights
  if (layer && warp < kWorkWarps) nw = ld_nc_v2(p.norm_weight + h0);
  float scale_l = 0.f, base_l = 0.f;  // the control warp's lane c: scale of c's group, base[c]
  if (coeff && warp == kCtl && lane < C) {
    scale_l = p.scale[lane < N ? 0 : (lane < 2 * N ? 1 : 2)];
    base_l = p.base[lane];
  }
  __syncthreads();

  // ---- 2. wait for the preceding kernel on the stream, then the row data
  griddep_wait();
  if (tid == 0 && exch) {
    const uint32_t e = ld_relaxed_gpu(p.ctl + kEpochWord);
    *tag_slot = e + 1u == 0u ? 1u : e + 1u;
  }
  auto issue_chunk = [&](int c) {  // one thread; MoE gathers are issued by the whole warp below
    const int s = c % S;
    unsigned char* dst = st_s + s * L.stage_bytes;
    mbar_arrive_expect_tx(&full[s], L.stage_bytes);
    if constexpr (FRONT == kPartials) {
      tma_load_3d(dst, &tm_x, g * kCols, c * kRC, 0, &full[s]);
    } else if constexpr (FRONT == kBroadcast) {
      tma_load_2d(dst, &tm_x, g * kCols, c * kRC, &full[s]);
    }
    if constexpr (FRONT != kBroadcast) tma_load_3d(dst + L.res_units * 128, &tm_res, g * kCols, 0, c * kRC, &full[s]);
  };
  auto issue_moe_chunk = [&](int c) {  // the control warp
    const int s = c % S;
    unsigned char* dst = st_s + s * L.stage_bytes;
    const int K = p.topk;
    if (lane == 0) {
      const int gathered = p.num_perm > 0 ? K * kRC * 128 : 0;
      mbar_arrive_expect_tx(&full[s], L.stage_bytes - (K * kRC * 128 - gathered));
      tma_load_2d(dst + K * kRC * 128, &tm_x, g * kCols, c * kRC, &full[s]);  // shared output
      tma_load_3d(dst + L.res_units * 128, &tm_res, g * kCols, 0, c * kRC, &full[s]);
    }
    __syncwarp();
    if (p.num_perm > 0) {
      for (int qq = lane; qq < K * 4; qq += 32) {  // slot t, rows 4*quad .. 4*quad + 3 of the chunk
        const int t = qq >> 2, quad = qq & 3;
        int idx[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = c * kRC + quad * 4 + i;
          const int e = r < R ? e2p_s[r * K + t] : 0;
          idx[i] = (e >= 0 && e < p.num_perm) ? e : 0;  // such slots add nothing below
        }
        tma_gather4(dst + (t * kRC + quad * 4) * 128, &tm_gather, g * kCols, idx[0], idx[1], idx[2], idx[3], &full[s]);
      }
    }
  };
  if (FRONT != kMoe && tid == kCtl * 32) {
    for (int c = 0; c < nch && c < S; ++c) issue_chunk(c);
  }
  for (int k = tid; k < R * MIX; k += kThreads) {  // [R][post n | comb n*n | pre n]
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
    for (int k = tid; k < R * p.topk; k += kThreads) {
      cp_async4(e2p_s + k, p.e2p + k);
      cp_async4(ew_s + k, p.ew + k);
    }
  }
  // the fn slice's three bf16 terms, while the row data is in flight: one thread
  // waits on the copy, the others block in the barrier (no issue slots)
  bool fn_ok = true;
  if (coeff) {
    const bool ok = tid == 0 ? mbar_wait_bounded(fnbar, 0, deadline) : true;
    fn_ok = __syncthreads_and(ok) != 0;
    if (!fn_ok && tid == 0) record_error(status, MHC_ERR_DEVICE_TIMEOUT);
    if (fn_ok && !packed) {
      // consecutive threads take consecutive fn columns: conflict-free reads of the
      // fp32 slice [kin][C]
      for (int it = tid; it < N * C * 8; it += kThreads) {
        const int c = it % C, rest = it / C;
        const int oct = rest & 7, j = rest >> 3;
        split_octet<N>(reinterpret_cast<const float*>(fst_s + j * kCols * C * 4), a_s + j * AR * 128, c, oct);
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();  // the mixes (and MoE routing) staged, the fn terms complete
  const uint32_t tag = exch ? *tag_slot : 0u;
  if (FRONT == kMoe && warp == kCtl) {
    for (int c = 0; c < nch && c < S; ++c) issue_moe_chunk(c);
  }

  if (warp < kWorkWarps) {
    // ---- 3. the chunks of group q: x, post-mix, new streams, staged streams, row sums
    // with one stage, group 0 takes every chunk in order (two groups on one stage
    // could each see the other's phase of its barrier as their own)
    const int c0 = S > 1 ? q : (q == 0 ? 0 : nch), cstep = S > 1 ? 2 : 1;
    for (int c = c0; c < nch; c += cstep) {
      const int s = c % S;
      // one lane of the group waits for the chunk's data; the group blocks in its barrier
      if (wq == 0 && lane == 0 && !mbar_wait_bounded(&full[s], (c / S) & 1, deadline))
        record_error(status, MHC_ERR_DEVICE_TIMEOUT);
      named_sync_group(q);
      const int r = c * kRC + rl;
      const bool valid = r < R;
      const unsigned char* sp = st_s + s * L.stage_bytes;
      const float* mix = mix_s + (valid ? r : 0) * MIX;
      float2 nf[N][2];  // the new streams, as rounded to bf16
      uint2 nb[N];
      float2 xs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      if constexpr (FRONT == kPartials || FRONT == kMoe || lane_partials(FRONT)) {
        if constexpr (FRONT == kPartials) {
          for (int u = 0; u < p.P; ++u) {  // the partials in order
            float2 f[2];
            unpack4x2(lds_v2(sp + (u * kRC + rl) * 128 + v * 8), f);
#pragma unroll
            for (int t = 0; t < 2; ++t) xs[t] = __fadd2_rn(xs[t], f[t]);
          }
        } else if constexpr (FRONT == kMoe) {
          unpack4x2(lds_v2(sp + (p.topk * kRC + rl) * 128 + v * 8), xs);  // shared output first
          if (valid) {
            const int* idx = e2p_s + r * p.topk;
            const float* wt = ew_s + r * p.topk;
            for (int u = 0; u < p.topk; ++u) {  // then the top_k slots in order
              const int e = idx[u];
              if (e >= p.num_perm) {
                if (v == 0) record_error(status, MHC_ERR_DEVICE_INDEX);
              } else if (e >= 0) {
                float2 f[2];
                unpack4x2(lds_v2(sp + (u * kRC + rl) * 128 + v * 8), f);
                const float2 w2 = make_float2(wt[u], wt[u]);
#pragma unroll
                for (int t = 0; t < 2; ++t) xs[t] = __ffma2_rn(w2, f[t], xs[t]);
              }
            }
          }
        } else {  // lane-read partials: a table of (peer) pointers, or mailbox slots
          if (valid) {
            const size_t off = static_cast<size_t>(r) * H + h0;
            for (int u = 0; u < p.P; ++u) {
              const __nv_bfloat16* src = p.pptr[u] + off;
              uint2 w = ld_cg_v2(src);
              if (FRONT == kMailbox) {
                while (has_neg_zero(w)) {  // re-read until its producer has written every element
                  if (clock64() > deadline) {
                    record_error(status, MHC_ERR_DEVICE_TIMEOUT);
                    break;
                  }
                  w = ld_volatile_v2(src);
                }
              }
              float2 f[2];
              unpack4x2(w, f);
#pragma unroll
              for (int t = 0; t < 2; ++t) xs[t] = __fadd2_rn(xs[t], f[t]);
            }
            if (FRONT == kMailbox) {  // consumed: back to "not written" for the round after next
              for (int u = 0; u < p.P; ++u)
                st_v2(const_cast<__nv_bfloat16*>(p.pptr[u]) + off, make_uint2(kNegZero2, kNegZero2));
            }
          }
        }
        float2 rf[N][2];
#pragma unroll
        for (int j = 0; j < N; ++j) unpack4x2(lds_v2(sp + (L.res_units + rl * N + j) * 128 + v * 8), rf[j]);
        // mHC post: new[i] = bf16(post[i] * x + sum_j comb[j][i] * res[j]), column
        // pairs in packed f32x2 arithmetic (per element the same fp32 operations,
        // in the same order, as one at a time)
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
      } else if constexpr (FRONT == kStreams) {
#pragma unroll
        for (int j = 0; j < N; ++j) {
          nb[j] = lds_v2(sp + (rl * N + j) * 128 + v * 8);
          unpack4x2(nb[j], nf[j]);
        }
      } else {  // kBroadcast: every stream is the embedding row
        const uint2 xv = lds_v2(sp + rl * 128 + v * 8);
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
        unsigned aw[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          float2 m = nf[0][t];
#pragma unroll
          for (int j = 1; j < N; ++j) m = __fadd2_rn(m, nf[j][t]);
          m = __fmul2_rn(m, make_float2(kInvN, kInvN));
          aw[t] = pack_bf16x2(m.x, m.y);
        }
        st_v2(p.aux_out + static_cast<size_t>(r) * H + h0, make_uint2(aw[0], aw[1]));
      }
      if (exch) {  // the new streams staged for the projection and the layer input
#pragma unroll
        for (int i = 0; i < N; ++i)
          *reinterpret_cast<uint2*>(v_s + i * L.r_alloc * 128 + sw128_offset(r, v)) = nb[i];
      }
      if (layer) {  // collapse with the carried pre (identity pre-mix for the broadcast)
        float2 sq = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          float2 cc;
          if (FRONT == kBroadcast) {
            cc = xs[t];
          } else {
            cc = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < N; ++j) {
              const float pj = mix[N + N * N + j];
              cc = __ffma2_rn(make_float2(pj, pj), nf[j][t], cc);
            }
          }
          sq = __ffma2_rn(cc, cc, sq);
        }
        const float sc2 = sum16_lanes(sq.x + sq.y);
        if (valid && v == 0) rec_s[r * kRecF + C + 1] = sc2;
      }
      if (coeff) {  // sum of v^2 of the row's streams, then the chunk's projection
        float2 sv = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
          for (int t = 0; t < 2; ++t) sv = __ffma2_rn(nf[i][t], nf[i][t], sv);
        const float sv2 = sum16_lanes(sv.x + sv.y);
        if (valid && v == 0) rec_s[r * kRecF + C] = sv2;
        named_sync_group(q);  // the group's rows of the chunk staged; its stage read
        float* part = L.part_off >= 0 ? reinterpret_cast<float*>(smem + L.part_off + q * part_bytes(N))
                                      : reinterpret_cast<float*>(st_s + s * L.stage_bytes);
        if (fn_ok) project_chunk<N>(a_s, v_s, L.r_alloc, c, wq, lane, part);
        named_sync_group(q);
        const int kw = 4 * N < kGroupWarps ? 4 * N : kGroupWarps;  // warps that ran K steps
        for (int it = wq * 32 + lane; it < kRC * C; it += kGroupWarps * 32) {  // partials added in warp order
          const int rr = it / C, col = it - rr * C;
          if (c * kRC + rr < R) {
            float a = 0.f;
            for (int w = 0; w < kw; ++w) a += part[(w * kRC + rr) * C + col];
            rec_s[(c * kRC + rr) * kRecF + col] = a;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&vready[c]);
    }
  } else {
    // ---- 4. the control warp: a stage is refilled once its chunk is done
    for (int c = 0; c + S < nch; ++c) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(&vready[c], 0, deadline);
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        if (lane == 0) record_error(status, MHC_ERR_DEVICE_TIMEOUT);
        break;  // the chunks not refilled run out of their own waits
      }
      if constexpr (FRONT == kMoe) {
        issue_moe_chunk(c + S);
      } else {
        if (lane == 0) issue_chunk(c + S);
      }
      __syncwarp();
    }
  }

  if (exch) {
    // ---- 5. publish this CTA's row records as tagged words at rec[g][r][f]: one
    // contiguous run per CTA
    __syncthreads();  // every row's records complete
    for (int it = tid; it < R * NFP; it += kThreads) {
      const int r = it / NFP, f = it - r * NFP;
      const bool has = f <= C ? coeff : (f == C + 1 && layer);
      st_tagged(p.rec + static_cast<size_t>(g) * R * NFP + it, tag, has ? rec_s[r * kRecF + f] : 0.f);
    }
    griddep_launch_dependents();  // this boundary's HBM stream is done: the next may start its set-up

    // ---- 6. CTA g adds up rows g, g + G, ...: their records from every CTA, read
    // as 16-byte pairs of words (all of a record with the coefficients, else the
    // pair holding sum c^2), each field summed over the CTAs by 8 lanes
    const int nslot = g < R ? (R - 1 - g) / G + 1 : 0;
    if (nslot > 0) {
      constexpr int B = 8;
      const int kc0 = coeff ? 0 : (C + 1) / 2, nk = coeff ? NFP / 2 : 1;
      float* gb = reinterpret_cast<float*>(st_s);  // [slot][G][NFP] the records' values
      const int total = nslot * G * nk;
      auto chunk = [&](int i) -> const unsigned long long* {
        const int slot = i / (G * nk), rem = i - slot * G * nk;
        const int gg = rem / nk, k = kc0 + rem - gg * nk;
        return p.rec + (static_cast<size_t>(gg) * R + g + slot * G) * NFP + 2 * k;
      };
      for (int i0 = tid; i0 < total; i0 += B * kThreads) {
        ulonglong2 w[B];
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (i0 + b * kThreads < total) w[b] = ld_tagged2(chunk(i0 + b * kThreads));
        while (true) {  // the stale pairs re-read together until they carry the tag (bounded)
          bool all = true;
#pragma unroll
          for (int b = 0; b < B; ++b)
            if (i0 + b * kThreads < total && (tag_of(w[b].x) != tag || tag_of(w[b].y) != tag)) all = false;
          if (all) break;
          if (clock64() > deadline) {
            record_error(status, MHC_ERR_DEVICE_TIMEOUT);
            break;
          }
#pragma unroll
          for (int b = 0; b < B; ++b)
            if (i0 + b * kThreads < total && (tag_of(w[b].x) != tag || tag_of(w[b].y) != tag))
              w[b] = ld_tagged2(chunk(i0 + b * kThreads));
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int i = i0 + b * kThreads;
          if (i < total) {
            const int slot = i / (G * nk), rem = i - slot * G * nk;
            const int gg = rem / nk, k = kc0 + rem - gg * nk;
            float* d = gb + (slot * G + gg) * NFP + 2 * k;
            d[0] = value_of(w[b].x);
            d[1] = value_of(w[b].y);
          }
        }
      }
      __syncthreads();
      const int f0 = coeff ? 0 : C + 1, nf = (layer ? C + 2 : C + 1) - f0;
      const int units = nslot * nf;
      const int gs = (G + 7) / 8;
      for (int u0 = 0; u0 < units; u0 += kThreads / 8) {
        if (u0 + warp * 4 >= units) continue;  // (warp-uniform) no unit for this warp
        const int u = u0 + tid / 8, pp = tid & 7;
        // every lane of the warp takes part in the butterfly
        const bool active = u < units;
        const int uu = active ? u : 0;
        const int slot = uu / nf, f = f0 + uu - slot * nf;
        const float* col = gb + slot * G * NFP + f;
        float sum = 0.f;
        const int ge = (pp + 1) * gs < G ? (pp + 1) * gs : G;
        if (active)
          for (int gg = pp * gs; gg < ge; ++gg) sum += col[gg * NFP];  // lane pp: CTAs pp*gs .. in order
#pragma unroll
        for (int m = 1; m <= 4; m <<= 1) sum += __shfl_xor_sync(kFull, sum, m);
        if (active && pp == 0) cft_s[slot * kRecF + f] = sum;
      }
      __syncthreads();
      if (layer) {  // the rows' sums c^2, one copy for every CTA: tot[c][r]
        for (int it = tid; it < nslot * G; it += kThreads) {
          const int sl = it / G, c = it - sl * G;
          st_tagged(p.tot + static_cast<size_t>(c) * R + g + sl * G, tag, cft_s[sl * kRecF + C + 1]);
        }
      }
    }
    if (warp == kCtl && coeff) {
      for (int sl = 0; sl < nslot; ++sl)
        coefficient_row<N>(p, g + sl * G, cft_s + sl * kRecF, scale_l, base_l, lane);
    }
    if (warp < kWorkWarps && layer) {
      // every row's sum c^2, from this CTA's copy
      for (int r = tid; r < R; r += kWorkThreads) {
        const unsigned long long* src = p.tot + static_cast<size_t>(g) * R + r;
        unsigned long long w = ld_tagged(src);
        while (tag_of(w) != tag) {
          if (clock64() > deadline) {
            record_error(status, MHC_ERR_DEVICE_TIMEOUT);
            break;
          }
          w = ld_tagged(src);
        }
        inv_s[r] = rsqrtf(__fdiv_rn(value_of(w), static_cast<float>(H)) + p.norm_eps);
      }
      named_sync_workers();
    }
    if (warp < kWorkWarps && layer) {
      // ---- 7. the layer input (and MXFP8) of this CTA's columns, rows 2 * warp +
      // lane / 16 of each 32-row pass, the lane's 4 columns
      const int scols = H / 32;
      const int col_tiles = (scols + 3) / 4;
      float2 wv[2];
      unpack4x2(nw, wv);
      for (int r0 = 0; r0 < R; r0 += 2 * kWorkWarps) {
        // every lane takes part in the block shuffles; rows past R store nothing
        const int r = r0 + warp * 2 + (lane >> 4);
        const bool valid = r < R;
        const int rr = valid ? r : 0;
        const float* mix = mix_s + rr * MIX;
        // the collapse recomputed from the staged bf16 streams exactly as its squares were summed
        float2 cc[2];
        if (FRONT == kBroadcast) {
          unpack4x2(lds_v2(v_s + sw128_offset(rr, v)), cc);
        } else {
          cc[0] = cc[1] = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < N; ++j) {
            float2 f[2];
            unpack4x2(lds_v2(v_s + j * L.r_alloc * 128 + sw128_offset(rr, v)), f);
            const float pj = mix[N + N * N + j];
#pragma unroll
            for (int t = 0; t < 2; ++t) cc[t] = __ffma2_rn(make_float2(pj, pj), f[t], cc[t]);
          }
        }
        const float inv = inv_s[rr];
        const float y[4] = {cc[0].x * inv * wv[0].x, cc[0].y * inv * wv[0].y, cc[1].x * inv * wv[1].x,
                            cc[1].y * inv * wv[1].y};
        const uint2 yb = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
        if (valid) st_v2(p.layer_input + static_cast<size_t>(r) * H + h0, yb);
        if (p.q_data != nullptr) {
          float2 yr[2];
          unpack4x2(yb, yr);
          const float ys[4] = {yr[0].x, yr[0].y, yr[1].x, yr[1].y};
          float amax = 0.f;
          bool finite = true;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            amax = fmaxf(amax, fabsf(ys[e]));
            finite = finite && isfinite(ys[e]);
          }
          // the 8 lanes of a 32-column block: lanes sharing lane bits 3 and 4
#pragma unroll
          for (int m = 1; m <= 4; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));
          const unsigned fin = __ballot_sync(kFull, finite);
          const bool grp_ok = ((fin >> (lane & 24)) & 0xffu) == 0xffu;
          unsigned d;
          unsigned char sbyte;
          if (grp_ok) {
            const int e = e8m0_exponent(amax);
            const float sc8 = exp2_neg(e);
            d = static_cast<unsigned>(e4m3x2(ys[0] * sc8, ys[1] * sc8)) |
                (static_cast<unsigned>(e4m3x2(ys[2] * sc8, ys[3] * sc8)) << 16);
            sbyte = static_cast<unsigned char>(e + 127);
          } else {
            d = 0x7f7f7f7fu;
            sbyte = 0xff;
          }
          if (valid) *reinterpret_cast<unsigned*>(p.q_data + static_cast<size_t>(r) * H + h0) = d;
          if (valid && (v & 7) == 0) {
            const int sc32 = h0 / 32;
            p.q_scale[p.q_swizzled ? swizzled_scale_offset(r, sc32, col_tiles) : r * scols + sc32] = sbyte;
          }
        }
      }
      if (p.q_data != nullptr && p.q_swizzled) {
        // the padding of the swizzled scale buffer, spread over every CTA: rows R..
        // whole, then the padding columns of rows below R
        const int rows_p = (R + 127) & ~127;
        const int pad_cols = col_tiles * 4 - scols;
        const int n_rows = (rows_p - R) * col_tiles * 4;
        const int n_cols = R * pad_cols;
        for (int k = g * kWorkThreads + tid; k < n_rows + n_cols; k += G * kWorkThreads) {
          if (k < n_rows) {
            const int r = R + k / (col_tiles * 4), u = k % (col_tiles * 4);
            p.q_scale[swizzled_scale_offset(r, u, col_tiles)] = 0;
          } else {
            const int kk = k - n_rows;
            const int r = kk / pad_cols, sc32 = scols + kk % pad_cols;
            p.q_scale[swizzled_scale_offset(r, sc32, col_tiles)] = 0;
          }
        }
      }
    }
    // CTA 0 has read row 0's records from every CTA, so every CTA of this launch
    // has read the epoch: the next launch may use the next tag.
    if (g == 0 && tid == 0) p.ctl[kEpochWord] = tag;
  } else {
    griddep_launch_dependents();
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
  for (int k = threadIdx.x * 8; k < q.H; k += blockDim.x * 8) {
    uint4 v = ld_nc_v4(src + k);
    v.x = clear_neg_zero2(v.x);
    v.y = clear_neg_zero2(v.y);
    v.z = clear_neg_zero2(v.z);
    v.w = clear_neg_zero2(v.w);
    st_v4(slot + k, v);
  }
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


// fn [n*H, C] fp32 -> per CTA g the A operand image of its projection, the
// bytes the kernel would build in shared memory: [n atom columns][arows][128 B],
// row t*C + c holding term t of fn column c over the 64 K values of stream j
// (fn row j*H + 64g + kin), 16-byte chunks XOR-swizzled by row; rows >= 3C zero.
template <int N>
__global__ void __launch_bounds__(256) pack_projection_kernel(const float* __restrict__ fn, int H,
                                                              unsigned char* __restrict__ out) {
  constexpr int C = logits_of(N);
  constexpr int AR = arows_of(N);
  const int g = blockIdx.x;
  unsigned char* dst = out + static_cast<size_t>(g) * aimage_bytes(N);
  for (int it = threadIdx.x; it < N * AR * 8; it += blockDim.x) {
    const int oct = it & 7, jm = it >> 3;
    const int m = jm % AR, j = jm / AR;
    unsigned w[4] = {0u, 0u, 0u, 0u};
    if (m < 3 * C) {
      const int t = m / C, c = m - t * C;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float f = fn[(static_cast<size_t>(j) * H + g * kCols + oct * 8 + e) * C + c];
        __nv_bfloat16 term[3];
        split3(f, term[0], term[1], term[2]);
        w[e >> 1] |= static_cast<unsigned>(__bfloat16_as_ushort(term[t])) << ((e & 1) * 16);
      }
    }
    *reinterpret_cast<uint4*>(dst + j * AR * 128 + m * 128 + (((oct ^ m) & 7) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
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
// Host side: argument checks, tensor maps, launch configuration, C ABI
// =====================================================================================

namespace {

using namespace mhc;

int64_t g_budget_ns = 1000000000LL;
int g_extra_tx = 0;

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace bytes: the header, then [G][R][fields] and [R] tagged words.
size_t ws_layout(int R, int H, int n) {
  const size_t G = static_cast<size_t>(H / kCols);
  return kWsHeader + static_cast<size_t>(fields_of(n) + 1) * G * static_cast<size_t>(R) * 8;
}

// The workspace's parts for a call of p.R rows over p.H columns.
void set_workspace(Params& p, void* ws, int n) {
  p.ctl = static_cast<unsigned*>(ws);
  p.rec = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + kWsHeader);
  p.tot = p.rec + static_cast<size_t>(p.H / kCols) * p.R * fields_of(n);
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

// A bf16 tensor map of `rank` dimensions (innermost first), strides in bytes of
// dimensions 1.., box sizes; no swizzle, out-of-range elements read as zero.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t d[3], s[2];
  cuuint32_t b[3], e[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides[i];
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, s, b, e,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// What the host needs beyond Params to build a launch's tensor maps.
struct Sources {
  const __nv_bfloat16* partials = nullptr;  // kPartials: [P] x [R, H] with a stride
  int64_t partial_stride = 0;
  const __nv_bfloat16* residual = nullptr;  // [R, n, H]
  const __nv_bfloat16* rows2d = nullptr;    // kBroadcast: x [R, H]; kMoe: shared_output [R, H]
};

// ---------------------------------------------------------------- launch

constexpr int kSmemMax = 227 * 1024;  // the largest dynamic shared memory a block may have

std::mutex g_cfg_mu;
// (kernel, device, grid, smem bytes) -> whether every CTA of the grid can be resident
std::map<std::tuple<const void*, int, int, int>, bool> g_fit;

// The kernel's shared-memory limit and carveout, set once per kernel and device.
std::map<std::pair<const void*, int>, bool> g_configured;

template <typename Kern>
bool configure(Kern kern, int dev) {
  const auto key = std::make_pair(reinterpret_cast<const void*>(kern), dev);
  std::lock_guard<std::mutex> lock(g_cfg_mu);
  if (g_configured.count(key)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           static_cast<int>(cudaSharedmemCarveoutMaxShared)) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  g_configured[key] = true;
  return true;
}

// Whether all `grid` CTAs can be resident at once (every CTA waits, bounded, for
// the others' published records).
template <typename Kern>
bool blocks_fit(Kern kern, int dev, int grid, int smem) {
  const auto key = std::make_tuple(reinterpret_cast<const void*>(kern), dev, grid, smem);
  {
    std::lock_guard<std::mutex> lock(g_cfg_mu);
    auto it = g_fit.find(key);
    if (it != g_fit.end()) return it->second;
  }
  int per_sm = 0, sms = 0;
  const bool ok = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) == cudaSuccess &&
                  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
                  per_sm * sms >= grid;
  (void)cudaGetLastError();
  std::lock_guard<std::mutex> lock(g_cfg_mu);
  g_fit[key] = ok;
  return ok;
}

template <int N, int FRONT>
mhc_status launch_boundary(Params& p, const Sources& src, cudaStream_t stream) {
  const int G = p.H / kCols;
  const int R = p.R;
  const bool coeff = p.do_coeff != 0, layer = p.do_layer != 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MHC_ERR_CUDA;
  auto kern = boundary_kernel<N, FRONT>;
  if (!configure(kern, dev)) return MHC_ERR_CUDA;
  p.extra_tx = g_extra_tx;
  p.budget_ns = g_budget_ns;

  // tensor maps of this call's buffers (the maps are kernel parameters, so a
  // captured graph keeps them)
  CUtensorMap maps[3];
  std::memset(maps, 0, sizeof(maps));
  const uint64_t H = static_cast<uint64_t>(p.H);
  if (FRONT == kPartials) {
    const uint64_t pstride = p.P > 1 ? static_cast<uint64_t>(src.partial_stride) * 2 : static_cast<uint64_t>(R) * H * 2;
    const uint64_t dims[3] = {H, static_cast<uint64_t>(R), static_cast<uint64_t>(p.P)};
    const uint64_t strides[2] = {H * 2, pstride};
    const uint32_t box[3] = {kCols, kRC, static_cast<uint32_t>(p.P)};
    if (!make_map(&maps[0], src.partials, 3, dims, strides, box)) return MHC_ERR_CUDA;
  }
  if (FRONT == kBroadcast || FRONT == kMoe) {
    const uint64_t dims[2] = {H, static_cast<uint64_t>(R)};
    const uint64_t strides[1] = {H * 2};
    const uint32_t box[2] = {kCols, kRC};
    if (!make_map(&maps[0], src.rows2d, 2, dims, strides, box)) return MHC_ERR_CUDA;
  }
  if (FRONT != kBroadcast) {
    const uint64_t dims[3] = {H, static_cast<uint64_t>(N), static_cast<uint64_t>(R)};
    const uint64_t strides[2] = {H * 2, H * 2 * N};
    const uint32_t box[3] = {kCols, static_cast<uint32_t>(N), kRC};
    if (!make_map(&maps[1], src.residual, 3, dims, strides, box)) return MHC_ERR_CUDA;
  }
  if (FRONT == kMoe && p.num_perm > 0) {
    const uint64_t dims[2] = {H, static_cast<uint64_t>(p.num_perm)};
    const uint64_t strides[1] = {H * 2};
    const uint32_t box[2] = {kCols, 1};
    if (!make_map(&maps[2], p.gemm2, 2, dims, strides, box)) return MHC_ERR_CUDA;
  }

  // stages in flight: as many as the chunks need and shared memory holds, with
  // every CTA of the grid resident
  const int nch = (R + kRC - 1) / kRC;
  int smem = 0;
  p.stages = 0;
  for (int st = nch < kMaxStages ? nch : kMaxStages; st >= 1; --st) {
    // a stage that is refilled serves one group only: an even count, or one stage
    // and one group
    if (st < nch && st % 2 == 1 && st != 1) continue;
    const Layout L = layout_of<N>(FRONT, R, G, p.P, p.topk, coeff, layer, st, p.fn_packed != nullptr);
    const int bytes = L.total + 1024;
    if (bytes > kSmemMax || !blocks_fit(kern, dev, G, bytes)) continue;
    smem = bytes;
    p.stages = st;
    break;
  }
  if (p.stages == 0) return MHC_ERR_UNSUPPORTED_SHAPE;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p, maps[0], maps[1], maps[2]) != cudaSuccess) {
    (void)cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  return MHC_OK;
}

template <int FRONT>
mhc_status dispatch_n(Params& p, const Sources& src, int n, cudaStream_t s) {
  switch (n) {
    case 1: return launch_boundary<1, FRONT>(p, src, s);
    case 2: return launch_boundary<2, FRONT>(p, src, s);
    case 4: return launch_boundary<4, FRONT>(p, src, s);
    default: return MHC_ERR_UNSUPPORTED_SHAPE;
  }
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

// Checks and fills the layer input, MXFP8, coefficients and workspace shared by
// the full-boundary entry points.
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
  if (!ws || !aligned(ws, 256) || ws_bytes < ws_layout(R, H, n)) return MHC_ERR_WORKSPACE;
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
    p.fn_packed = static_cast<const unsigned char*>(coeffs->fn_packed);
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
  set_workspace(p, ws, n);
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
  return ws_layout(rows, hidden, hc_mult);
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

// mhc_boundary_post_pre over a table of partial pointers (checked by the callers):
// the lanes load the partials themselves (peer memory, or mailbox slots).
mhc_status post_pre_table(const __nv_bfloat16* const* pptr, int num_partials, const mhc_bf16* residual,
                          const float* post, const float* comb, const float* pre, const mhc_bf16* norm_weight,
                          float norm_eps, const mhc_coeff_args* coeffs, mhc_bf16* residual_out, mhc_bf16* aux_out,
                          mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8, float* post_out, float* comb_out,
                          float* pre_out, int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes,
                          mhc_stream stream, bool mailbox) {
  mhc_status st = check_mixes(residual, post, comb, residual_out);
  if (st != MHC_OK) return st;
  Params p{};
  for (int u = 0; u < num_partials; ++u) p.pptr[u] = pptr[u];
  p.premote = 1;
  p.P = num_partials;
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
  Sources src;
  src.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  return mailbox ? dispatch_n<kMailbox>(p, src, hc_mult, stream) : dispatch_n<kTable>(p, src, hc_mult, stream);
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
  if (num_partials > 1 && partial_stride < 0) {  // not a tensor map: the lanes load the partials
    const __nv_bfloat16* pptr[kMaxPartials];
    for (int u = 0; u < num_partials; ++u)
      pptr[u] = reinterpret_cast<const __nv_bfloat16*>(partials) + static_cast<int64_t>(u) * partial_stride;
    return post_pre_table(pptr, num_partials, residual, post, comb, pre, norm_weight, norm_eps, coeffs, residual_out,
                          aux_out, layer_input, mxfp8, post_out, comb_out, pre_out, rows, hidden, hc_mult, workspace,
                          ws_bytes, stream, false);
  }
  mhc_status st = check_mixes(residual, post, comb, residual_out);
  if (st != MHC_OK) return st;
  Params p{};
  p.P = num_partials;
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
  Sources src;
  src.partials = reinterpret_cast<const __nv_bfloat16*>(partials);
  src.partial_stride = partial_stride;
  src.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  return dispatch_n<kPartials>(p, src, hc_mult, stream);
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
  return post_pre_table(pptr, num_partials, residual, post, comb, pre, norm_weight, norm_eps, coeffs, residual_out,
                        aux_out, layer_input, mxfp8, post_out, comb_out, pre_out, rows, hidden, hc_mult, workspace,
                        ws_bytes, stream, false);
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
  mhc_status st = post_pre_table(pptr, world, residual, post, comb, pre, norm_weight, norm_eps, coeffs, residual_out,
                                 aux_out, layer_input, mxfp8, post_out, comb_out, pre_out, rows, hidden, hc_mult,
                                 workspace, ws_bytes, stream, true);
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
                                     float* post_out, float* comb_out, float* pre_out, int rows, int hidden,
                                     int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream) {
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
  if (pre == nullptr) {  // the residual-only form records gather-index errors in the workspace header
    if (!workspace || !aligned(workspace, 256) || ws_bytes < kWsHeader) return MHC_ERR_WORKSPACE;
    p.ctl = static_cast<unsigned*>(workspace);
  }
  Sources src;
  src.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  src.rows2d = reinterpret_cast<const __nv_bfloat16*>(shared_output);
  return dispatch_n<kMoe>(p, src, hc_mult, stream);
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
  if (num_partials > 1 && partial_stride < 0) {  // not a tensor map: the lanes load the partials
    for (int u = 0; u < num_partials; ++u)
      p.pptr[u] = reinterpret_cast<const __nv_bfloat16*>(partials) + static_cast<int64_t>(u) * partial_stride;
    p.premote = 1;
  }
  p.P = num_partials;
  p.post = post;
  p.comb = comb;
  p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
  p.write_res = 1;
  if (aux_out && !aligned(aux_out, 16)) return MHC_ERR_INVALID_ARG;
  p.aux_out = reinterpret_cast<__nv_bfloat16*>(aux_out);
  p.R = rows;
  p.H = hidden;
  Sources src;
  src.partials = reinterpret_cast<const __nv_bfloat16*>(partials);
  src.partial_stride = partial_stride;
  src.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  if (p.premote) return dispatch_n<kTable>(p, src, hc_mult, stream);
  return dispatch_n<kPartials>(p, src, hc_mult, stream);
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
  if (!workspace || !aligned(workspace, 256) || ws_bytes < ws_layout(rows, hidden, hc_mult)) return MHC_ERR_WORKSPACE;
  Params p{};
  p.R = rows;
  p.H = hidden;
  p.do_coeff = 1;
  p.fn = coeffs->fn;
  p.fn_packed = static_cast<const unsigned char*>(coeffs->fn_packed);
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
  set_workspace(p, workspace, hc_mult);
  if (layer_input) {
    if (!norm_weight || !aligned(norm_weight, 16) || !aligned(layer_input, 16) || !(norm_eps >= 0.f))
      return MHC_ERR_INVALID_ARG;
    p.do_layer = 1;
    p.norm_weight = reinterpret_cast<const __nv_bfloat16*>(norm_weight);
    p.norm_eps = norm_eps;
    p.layer_input = reinterpret_cast<__nv_bfloat16*>(layer_input);
  }
  Sources src;
  if (x) {
    if (pre_mix || !aligned(x, 16)) return MHC_ERR_INVALID_ARG;
    if (residual_out && !aligned(residual_out, 16)) return MHC_ERR_INVALID_ARG;
    p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
    p.write_res = residual_out != nullptr;
    src.rows2d = reinterpret_cast<const __nv_bfloat16*>(x);
    return dispatch_n<kBroadcast>(p, src, hc_mult, stream);
  }
  if (residual_out || !aligned(residual, 16)) return MHC_ERR_INVALID_ARG;
  if (layer_input && (!pre_mix || !aligned(pre_mix, 4))) return MHC_ERR_INVALID_ARG;
  p.pre = pre_mix;
  src.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  return dispatch_n<kStreams>(p, src, hc_mult, stream);
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
  const int pb = hc_mult == 1 ? aimage_bytes(1) : (hc_mult == 2 ? aimage_bytes(2) : aimage_bytes(4));
  return static_cast<size_t>(G) * pb;
}

mhc_status mhc_projection_pack(const float* fn, void* packed, int hidden, int hc_mult, mhc_stream stream) {
  if (!shape_ok(1, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!fn || !packed || !aligned(fn, 4) || !aligned(packed, 16)) return MHC_ERR_INVALID_ARG;
  const int G = hidden / kCols;
  unsigned char* out = static_cast<unsigned char*>(packed);
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
// 3,097,600 bytes: mhc_workspace_bytes(128, 7168, 4), the header, the row
// records [112 CTAs][128 rows][26 fields] and the totals [112 copies][128 rows]
constexpr size_t kNoAllocBytes =
    kWsHeader + static_cast<size_t>(fields_of(kNoAllocMaxHc) + 1) * (kNoAllocMaxHidden / kCols) * kNoAllocMaxRows * 8;
static_assert(kNoAllocBytes == 3097600, "the no-alloc scratch size");

// The array is zero at module load, as a workspace must be before first use
// (mhc_workspace_init): the status word, and the launch epoch that tags the
// row records every call rewrites.
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
      ws_layout(rows, hidden, hc_mult) > kNoAllocBytes)
    return MHC_ERR_WORKSPACE;  // needs more scratch than the fixed array holds
  void* ws = noalloc_scratch();
  if (ws == nullptr) return MHC_ERR_CUDA;
  return mhc_boundary_post_pre(partials, num_partials, partial_stride, residual, post, comb, pre, norm_weight,
                               norm_eps, coeffs, residual_out, aux_out, layer_input, mxfp8, post_out, comb_out,
                               pre_out, rows, hidden, hc_mult, ws, kNoAllocBytes, stream);
}

}  // extern "C"
