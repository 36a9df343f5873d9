// mHC decode boundary on B200 (sm_100a): the fused kernel and the C ABI of
// libmhc.so (declared in include/mhc.h).
//
// One launch does the whole boundary. Block g owns columns [64g, 64g+64) of H
// for every row, so each weight of fn is read from HBM exactly once:
//   1. TMA bulk copies bring the block's fn slice (n*64 rows of C floats) into
//      shared memory while the threads stream the partials (or the MoE gather)
//      and the residual streams with 128-bit loads;
//   2. per (row, 8 columns) a lane sums the partials, applies the mHC post-mix
//      (vllm ...boundary.boundary, Boundaries.post_only: mhc_post(x, residual,
//      post, comb)), rounds the new streams to bf16 and stores them, collapses
//      them with the carried pre (BoundaryState.pre) and accumulates, over its
//      32 stream values, sum c^2, sum v^2 and the C dot products with fn
//      (CUDA-core packed FMA);
//   3. the 8 lanes of a row reduce their sums (shuffle reduce-scatter) and the
//      block writes them to the workspace;
//   4. one bounded grid barrier; then every block normalises its own columns
//      into the layer input (and MXFP8), and block g finishes the coefficients
//      (logits, sigmoid, Sinkhorn in registers) of rows g, g+G, ...
// The residual-only variant stops after step 2 and needs no barrier.
// All reductions run in a fixed order, so results are bitwise reproducible.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mhc.h"
#include "mhc_device.cuh"

namespace mhc {

constexpr int kCols = 64;      // columns of H per block
constexpr int kThreads = 256;  // 8 warps; a warp covers 4 rows x 64 columns per step
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRows = 128;
constexpr int kMaxPartials = 16;
constexpr int kMaxTopK = 16;
constexpr int kMaxIters = 1000;
constexpr size_t kWsHeader = 1024;  // status, barrier count, barrier generation (own 128-B lines)
constexpr int kStatusWord = 0, kBarCountWord = 32, kBarGenWord = 64;

enum Front { kPartials = 0, kMoe = 1, kStreams = 2, kBroadcast = 3 };

__host__ __device__ constexpr int logits_of(int n) { return 2 * n + n * n; }
// Values reduced per row: C dot products, sum v^2, sum c^2, padded to a power of two >= 8.
__host__ __device__ constexpr int red_of(int n) {
  return logits_of(n) + 2 <= 8 ? 8 : (logits_of(n) + 2 <= 16 ? 16 : 32);
}
__host__ __device__ constexpr int fn_piece_bytes(int n) { return 8 * logits_of(n) * 4 + 16; }

struct Params {
  // front ends
  const __nv_bfloat16* partials;
  int64_t pstride;
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
  const float* scale;
  const float* base;
  float rms_eps, pre_eps, sk_eps, alpha;
  int iters;
  __nv_bfloat16* residual_out;
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
  int extra_arrivals;
  int64_t budget_ns;
};

struct SmemLayout {
  int fn_off, mix_off, c_off, moe_off, inv_off, red_off, bar_off, total;
};

template <int N>
__host__ __device__ inline SmemLayout smem_layout(int R, int topk, bool moe) {
  SmemLayout L{};
  int o = 0;
  L.fn_off = o;
  o += N * 8 * fn_piece_bytes(N);
  L.mix_off = o;
  o += R * (2 * N + N * N) * 4;
  o = (o + 15) & ~15;
  L.c_off = o;
  o += R * kCols * 4;
  L.moe_off = o;
  if (moe) o += R * topk * 8;
  o = (o + 15) & ~15;
  L.inv_off = o;
  o += kMaxRows * 4;
  L.red_off = o;
  o += (kThreads + 64) * 4;
  o = (o + 15) & ~15;
  L.bar_off = o;
  o += 16;
  L.total = o;
  return L;
}

// Reduce-scatter `v` (M values) over the 8 lanes that share lane bits 3-4:
// afterwards lane with (lane & 7) == q holds, in v[0 .. M/8), the sums of
// values [q*M/8, (q+1)*M/8) over the 8 lanes. Fixed order: deterministic.
template <int M>
__device__ __forceinline__ void reduce_scatter8(float (&v)[M], int vec) {
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const int mask = 4 >> s;
    const int half = M >> (s + 1);
    const bool up = (vec & mask) != 0;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float send = up ? v[k] : v[k + half];
      const float keep = up ? v[k + half] : v[k];
      v[k] = keep + __shfl_xor_sync(kFull, send, mask);
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

__device__ __forceinline__ int swizzled_scale_offset(int r, int c, int col_tiles) {
  const int tile = (r >> 7) * col_tiles + (c >> 2);
  const int rr = r & 127;
  return tile * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3);
}

template <int N, int FRONT>
__global__ void __launch_bounds__(kThreads, 1) boundary_kernel(const Params p) {
  constexpr int C = logits_of(N);
  constexpr int RED = red_of(N);
  constexpr int PIECE = fn_piece_bytes(N);
  extern __shared__ __align__(128) unsigned char smem[];
  const SmemLayout L = smem_layout<N>(p.R, p.topk, FRONT == kMoe);
  unsigned char* fn_s = smem + L.fn_off;
  float* mix_s = reinterpret_cast<float*>(smem + L.mix_off);
  float* c_s = reinterpret_cast<float*>(smem + L.c_off);
  int* e2p_s = reinterpret_cast<int*>(smem + L.moe_off);
  float* ew_s = reinterpret_cast<float*>(smem + L.moe_off) + p.R * p.topk;
  float* inv_s = reinterpret_cast<float*>(smem + L.inv_off);
  float* red_s = reinterpret_cast<float*>(smem + L.red_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  int* flag_s = reinterpret_cast<int*>(smem + L.bar_off + 8);

  const int g = blockIdx.x;
  const int G = gridDim.x;
  const int H = p.H;
  const int R = p.R;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rq = lane >> 3, vec = lane & 7;
  const int h0 = g * kCols + vec * 8;  // this lane's 8 columns
  const uint64_t deadline = global_ns() + static_cast<uint64_t>(p.budget_ns);
  unsigned* status = p.ctl + kStatusWord;

  // ---- 1. start the fn slice copy (one bulk copy per 8 rows, 16 B gap between pieces)
  if (p.do_coeff) {
    if (tid == 0) mbar_init(bar, 1);
    __syncthreads();
    if (warp == 0) {
      if (lane == 0) mbar_arrive_expect_tx(bar, N * kCols * C * 4);
      __syncwarp();
      for (int m = lane; m < N * 8; m += 32) {
        const int i = m >> 3, piece = m & 7;
        const float* src = p.fn + (static_cast<size_t>(i) * H + g * kCols + piece * 8) * C;
        bulk_g2s(fn_s + m * PIECE, src, 8 * C * 4, bar);
      }
    }
  }
  // ---- mixes (and MoE routing) of every row into shared memory
  {
    constexpr int MIX = 2 * N + N * N;
    for (int k = tid; k < R * MIX; k += kThreads) {
      const int r = k / MIX, c = k - r * MIX;
      float v = 0.f;
      if (c < N) {
        v = (FRONT == kStreams || FRONT == kBroadcast) ? 0.f : p.post[r * N + c];
      } else if (c < N + N * N) {
        v = (FRONT == kStreams || FRONT == kBroadcast) ? 0.f : p.comb[r * N * N + (c - N)];
      } else {
        v = (p.pre != nullptr) ? p.pre[r * N + (c - N - N * N)] : 0.f;
      }
      mix_s[k] = v;
    }
    if (FRONT == kMoe) {
      for (int k = tid; k < R * p.topk; k += kThreads) {
        e2p_s[k] = p.e2p[k];
        ew_s[k] = p.ew[k];
      }
    }
  }
  __syncthreads();

  bool fn_ready = false;
  bool aborted = false;
  const int nquads = (R + 3) >> 2;
  for (int q = warp; q < nquads; q += kWarps) {
    const int r = q * 4 + rq;
    const bool valid = r < R;
    const float* mix = mix_s + (valid ? r : 0) * (2 * N + N * N);

    // ---- 2a. front end: the new streams nf[i][t] (bf16 values held as floats)
    float nf[N][8];
    uint4 nb[N];
    float xs[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) xs[t] = 0.f;
    if (FRONT == kPartials || FRONT == kMoe) {
      uint4 rv[N];
      if (valid) {
#pragma unroll
        for (int j = 0; j < N; ++j) rv[j] = ld_v4(p.residual + (static_cast<size_t>(r) * N + j) * H + h0);
        if (FRONT == kPartials) {
          const __nv_bfloat16* base = p.partials + static_cast<size_t>(r) * H + h0;
          for (int p0 = 0; p0 < p.P; p0 += 8) {
            uint4 pv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              if (p0 + u < p.P) pv[u] = ld_nc_v4(base + (p0 + u) * p.pstride);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              if (p0 + u < p.P) {
                float f[8];
                unpack8(pv[u], f);
#pragma unroll
                for (int t = 0; t < 8; ++t) xs[t] += f[t];
              }
            }
          }
        } else {
          unpack8(ld_nc_v4(p.shared_out + static_cast<size_t>(r) * H + h0), xs);
          const int* idx = e2p_s + r * p.topk;
          const float* wt = ew_s + r * p.topk;
          for (int t0 = 0; t0 < p.topk; t0 += 8) {
            uint4 gv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int k = t0 + u;
              if (k < p.topk) {
                const int e = idx[k];
                if (e >= 0 && e < p.num_perm) {
                  gv[u] = ld_nc_v4(p.gemm2 + static_cast<size_t>(e) * H + h0);
                } else {
                  gv[u] = make_uint4(0, 0, 0, 0);
                  if (e >= p.num_perm && vec == 0) record_error(status, MHC_ERR_DEVICE_INDEX);
                }
              }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int k = t0 + u;
              if (k < p.topk) {
                const int e = idx[k];
                if (e >= 0 && e < p.num_perm) {
                  float f[8];
                  unpack8(gv[u], f);
                  const float w = wt[k];
#pragma unroll
                  for (int t = 0; t < 8; ++t) xs[t] = fmaf(w, f[t], xs[t]);
                }
              }
            }
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < N; ++j) rv[j] = make_uint4(0, 0, 0, 0);
      }
      // mHC post: new[i] = bf16(post[i] * x + sum_j comb[j][i] * res[j])
      float rf[N][8];
#pragma unroll
      for (int j = 0; j < N; ++j) unpack8(rv[j], rf[j]);
#pragma unroll
      for (int i = 0; i < N; ++i) {
        float a[8];
        const float po = mix[i];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          float s = po * xs[t];
#pragma unroll
          for (int j = 0; j < N; ++j) s = fmaf(mix[N + j * N + i], rf[j][t], s);
          a[t] = s;
        }
        nb[i] = round8(a, nf[i]);
      }
    } else if (FRONT == kStreams) {
#pragma unroll
      for (int j = 0; j < N; ++j) {
        nb[j] = valid ? ld_v4(p.residual + (static_cast<size_t>(r) * N + j) * H + h0) : make_uint4(0, 0, 0, 0);
        unpack8(nb[j], nf[j]);
      }
    } else {  // kBroadcast: every stream is the embedding row
      const uint4 xv = valid ? ld_nc_v4(p.x + static_cast<size_t>(r) * H + h0) : make_uint4(0, 0, 0, 0);
      unpack8(xv, xs);
#pragma unroll
      for (int j = 0; j < N; ++j) {
        nb[j] = xv;
#pragma unroll
        for (int t = 0; t < 8; ++t) nf[j][t] = xs[t];
      }
    }

    // ---- 2b. store the new streams
    if (p.write_res && valid) {
#pragma unroll
      for (int i = 0; i < N; ++i) st_v4(p.residual_out + (static_cast<size_t>(r) * N + i) * H + h0, nb[i]);
    }
    if (!p.do_layer && !p.do_coeff) continue;

    // ---- 2c. collapse with the carried pre (identity pre-mix for the broadcast)
    float sc2 = 0.f;
    if (p.do_layer) {
      float c[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (FRONT == kBroadcast) {
          c[t] = xs[t];
        } else {
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < N; ++j) s = fmaf(mix[N + N * N + j], nf[j][t], s);
          c[t] = s;
        }
        sc2 = fmaf(c[t], c[t], sc2);
      }
      float4* cs = reinterpret_cast<float4*>(c_s + (valid ? r : 0) * kCols);
      if (valid) {
        cs[vec] = make_float4(c[0], c[1], c[2], c[3]);
        cs[8 + vec] = make_float4(c[4], c[5], c[6], c[7]);
      }
    }

    if (p.do_coeff) {
      // ---- 2d. projection of this lane's 8N stream values onto the C fn columns
      if (!fn_ready) {
        // warp-uniform decision: every lane of the warp shuffles below
        const bool ok = __all_sync(kFull, mbar_wait_bounded(bar, 0, deadline));
        fn_ready = true;
        if (!ok) {
          if (lane == 0) record_error(status, MHC_ERR_DEVICE_TIMEOUT);
          aborted = true;
          break;
        }
      }
      float red[RED];
#pragma unroll
      for (int k = 0; k < RED; ++k) red[k] = 0.f;
      float sv2 = 0.f;
      if constexpr (C % 4 == 0) {
        float2 acc[C / 2];
#pragma unroll
        for (int k = 0; k < C / 2; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < N; ++i) {
          const unsigned char* piece = fn_s + (i * 8 + vec) * PIECE;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float v = nf[i][t];
            sv2 = fmaf(v, v, sv2);
            const float2 vv = make_float2(v, v);
            const float4* f = reinterpret_cast<const float4*>(piece + t * C * 4);
#pragma unroll
            for (int c4 = 0; c4 < C / 4; ++c4) {
              const float4 w = f[c4];
              acc[2 * c4] = __ffma2_rn(vv, make_float2(w.x, w.y), acc[2 * c4]);
              acc[2 * c4 + 1] = __ffma2_rn(vv, make_float2(w.z, w.w), acc[2 * c4 + 1]);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < C / 2; ++k) {
          red[2 * k] = acc[k].x;
          red[2 * k + 1] = acc[k].y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < N; ++i) {
          const unsigned char* piece = fn_s + (i * 8 + vec) * PIECE;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float v = nf[i][t];
            sv2 = fmaf(v, v, sv2);
            const float* f = reinterpret_cast<const float*>(piece + t * C * 4);
#pragma unroll
            for (int c = 0; c < C; ++c) red[c] = fmaf(v, f[c], red[c]);
          }
        }
      }
      red[C] = sv2;
      red[C + 1] = sc2;
      // ---- 3. reduce over the row's 8 lanes and publish this block's partial sums
      reduce_scatter8<RED>(red, vec);
      if (valid) {
        float* dst = p.dot_part + (static_cast<size_t>(r) * G + g) * RED + vec * (RED / 8);
#pragma unroll
        for (int k = 0; k < RED / 8; ++k) dst[k] = red[k];
        if (p.do_layer && vec == (C + 1) / (RED / 8)) p.sc2_part[r * G + g] = red[(C + 1) % (RED / 8)];
      }
    } else {
      // layer input only: reduce sum c^2 over the row's 8 lanes
#pragma unroll
      for (int m = 4; m >= 1; m >>= 1) sc2 += __shfl_xor_sync(kFull, sc2, m);
      if (valid && vec == 0) p.sc2_part[r * G + g] = sc2;
    }
  }
  if (!p.do_layer && !p.do_coeff) return;
  if (p.do_coeff && !fn_ready) {
    // a warp with no rows still waits for the copy in flight into shared memory
    if (!mbar_wait_bounded(bar, 0, deadline)) {
      record_error(status, MHC_ERR_DEVICE_TIMEOUT);
      aborted = true;
    }
  }
  if (__syncthreads_or(aborted)) return;  // block-uniform

  // ---- 4. all blocks' partial sums are in the workspace after this barrier
  if (!grid_barrier(p.ctl + kBarCountWord, p.ctl + kBarGenWord, G + p.extra_arrivals, status, deadline,
                    MHC_ERR_DEVICE_TIMEOUT, flag_s))
    return;

  if (p.do_layer) {
    // ---- 4a. per-row inverse RMS of the collapse, summed over blocks in a fixed order
    for (int r = warp; r < R; r += kWarps) {
      float s = 0.f;
      for (int k = lane; k < G; k += 32) s += __ldcg(p.sc2_part + r * G + k);
      s = warp_sum(s);
      if (lane == 0) inv_s[r] = rsqrtf(__fdiv_rn(s, static_cast<float>(H)) + p.norm_eps);
    }
    __syncthreads();
    // ---- 4b. layer input (and MXFP8) of this block's columns
    float w[8];
    unpack8(ld_nc_v4(p.norm_weight + h0), w);
    const int scols = H / 32;
    const int col_tiles = (scols + 3) / 4;
    for (int q = warp; q < nquads; q += kWarps) {
      const int r = q * 4 + rq;
      if (r >= R) continue;  // whole 4-lane MXFP8 groups share r: no shuffle crosses this
      const float4* cs = reinterpret_cast<const float4*>(c_s + r * kCols);
      const float4 c0 = cs[vec], c1 = cs[8 + vec];
      const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float inv = inv_s[r];
      float y[8], yr[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) y[t] = c[t] * inv * w[t];
      const uint4 yb = round8(y, yr);
      st_v4(p.layer_input + static_cast<size_t>(r) * H + h0, yb);
      if (p.q_data != nullptr) {
        float amax = 0.f;
        bool finite = true;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          amax = fmaxf(amax, fabsf(yr[t]));
          finite = finite && isfinite(yr[t]);
        }
        // the 4 lanes of a 32-column block are vec 0-3 or 4-7 of the same row
        amax = fmaxf(amax, __shfl_xor_sync(0xffu << (lane & 24), amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffu << (lane & 24), amax, 2));
        const unsigned fin_mask = __ballot_sync(0xffu << (lane & 24), finite);
        const unsigned grp = (fin_mask >> (lane & 28)) & 0xfu;
        uint2 d;
        unsigned char sbyte;
        if (grp == 0xfu) {
          const int e = e8m0_exponent(amax);
          const float s = exp2_neg(e);
          d.x = static_cast<unsigned>(e4m3x2(yr[0] * s, yr[1] * s)) |
                (static_cast<unsigned>(e4m3x2(yr[2] * s, yr[3] * s)) << 16);
          d.y = static_cast<unsigned>(e4m3x2(yr[4] * s, yr[5] * s)) |
                (static_cast<unsigned>(e4m3x2(yr[6] * s, yr[7] * s)) << 16);
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
    if (p.q_data != nullptr && p.q_swizzled) {
      // zero the padding of the swizzled scale buffer: rows R.. of this block's two
      // scale columns, and (last block) the padding columns of every row
      const int rows_p = (R + 127) & ~127;
      const int sc0 = g * 2;
      for (int k = tid; k < (rows_p - R) * 2; k += kThreads) {
        const int r = R + (k >> 1), sc = sc0 + (k & 1);
        p.q_scale[swizzled_scale_offset(r, sc, col_tiles)] = 0;
      }
      if (g == G - 1) {
        const int pad_cols = col_tiles * 4 - scols;
        for (int k = tid; k < rows_p * pad_cols; k += kThreads) {
          const int r = k / pad_cols, sc = scols + (k - r * pad_cols);
          p.q_scale[swizzled_scale_offset(r, sc, col_tiles)] = 0;
        }
      }
    }
  }

  if (p.do_coeff) {
    // ---- 4c. coefficients of rows g, g+G, ...: sum the blocks' partials in a fixed order
    float* tot_s = red_s + kThreads;  // [RED]
    float* lg_s = tot_s + 32;         // comb logits [N*N]
    for (int r = g; r < R; r += G) {
      __syncthreads();
      {
        const int v = tid % RED, sub = tid / RED;
        constexpr int SUBS = kThreads / RED;
        float s = 0.f;
        for (int k = sub; k < G; k += SUBS) s += __ldcg(p.dot_part + (static_cast<size_t>(r) * G + k) * RED + v);
        red_s[sub * RED + v] = s;
      }
      __syncthreads();
      if (tid < RED) {
        constexpr int SUBS = kThreads / RED;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < SUBS; ++k) s += red_s[k * RED + tid];
        tot_s[tid] = s;
      }
      __syncthreads();
      if (tid < C) {
        const float inv = rsqrtf(__fdiv_rn(tot_s[C], static_cast<float>(N * H)) + p.rms_eps);
        const int grp = tid < N ? 0 : (tid < 2 * N ? 1 : 2);
        const float l = p.scale[grp] * inv * tot_s[tid] + p.base[tid];
        if (tid < N) {
          p.pre_out[r * N + tid] = 1.f / (1.f + expf(-l)) + p.pre_eps;
        } else if (tid < 2 * N) {
          p.post_out[r * N + (tid - N)] = p.alpha / (1.f + expf(-l));
        } else {
          lg_s[tid - 2 * N] = l;
        }
      }
      __syncthreads();
      if (tid == 0) {
        // Sinkhorn in registers: M = exp(L - max L); rows then columns, iters times
        float M[N][N];
        float mx = lg_s[0];
#pragma unroll
        for (int k = 1; k < N * N; ++k) mx = fmaxf(mx, lg_s[k]);
#pragma unroll
        for (int j = 0; j < N; ++j)
#pragma unroll
          for (int i = 0; i < N; ++i) M[j][i] = expf(lg_s[j * N + i] - mx);
        for (int it = 0; it < p.iters; ++it) {
#pragma unroll
          for (int j = 0; j < N; ++j) {
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < N; ++i) s += M[j][i];
            const float rcp = __frcp_rn(s + p.sk_eps);
#pragma unroll
            for (int i = 0; i < N; ++i) M[j][i] *= rcp;
          }
#pragma unroll
          for (int i = 0; i < N; ++i) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < N; ++j) s += M[j][i];
            const float rcp = __frcp_rn(s + p.sk_eps);
#pragma unroll
            for (int j = 0; j < N; ++j) M[j][i] *= rcp;
          }
        }
#pragma unroll
        for (int j = 0; j < N; ++j)
#pragma unroll
          for (int i = 0; i < N; ++i) p.comb_out[(r * N + j) * N + i] = M[j][i];
      }
    }
  }
}

// MXFP8 of a bf16 [R, H] matrix: a lane quantises 8 columns, 4 lanes a block.
__global__ void __launch_bounds__(256) mxfp8_rows_kernel(const __nv_bfloat16* __restrict__ x, int R, int H,
                                                          uint8_t* __restrict__ data, uint8_t* __restrict__ scale,
                                                          int swizzled) {
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
int g_extra_arrivals = 0;

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
  return R >= 1 && R <= kMaxRows && H >= kCols && H % kCols == 0 && (n == 1 || n == 2 || n == 4);
}

mhc_status check_coeff(const mhc_coeff_args* a) {
  if (a == nullptr) return MHC_OK;
  if (!a->fn || !a->scale || !a->base) return MHC_ERR_INVALID_ARG;
  if (!aligned(a->fn, 16) || !aligned(a->scale, 4) || !aligned(a->base, 4)) return MHC_ERR_INVALID_ARG;
  if (!(a->rms_eps >= 0.f) || !(a->pre_eps >= 0.f) || !(a->sinkhorn_eps >= 0.f)) return MHC_ERR_INVALID_ARG;
  if (a->sinkhorn_iters < 0 || a->sinkhorn_iters > kMaxIters) return MHC_ERR_INVALID_ARG;
  return MHC_OK;
}

mhc_status check_mxfp8(const mhc_mxfp8_out* q) {
  if (q == nullptr) return MHC_OK;
  if (!q->data || !q->scale || !aligned(q->data, 8)) return MHC_ERR_INVALID_ARG;
  return MHC_OK;
}

template <int N, int FRONT>
mhc_status launch_boundary(Params& p, cudaStream_t stream) {
  const SmemLayout L = smem_layout<N>(p.R, p.topk, FRONT == kMoe);
  auto kern = boundary_kernel<N, FRONT>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MHC_ERR_CUDA;
  static int configured[64] = {0};
  if (dev < 64 && configured[dev] < L.total) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
      return MHC_ERR_CUDA;
    configured[dev] = 200 * 1024;
  }
  const bool needs_barrier = p.do_layer || p.do_coeff;
  p.extra_arrivals = g_extra_arrivals;
  p.budget_ns = g_budget_ns;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.H / kCols);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = needs_barrier ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return MHC_ERR_UNSUPPORTED_SHAPE;
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  return MHC_OK;
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

mhc_status mhc_boundary_post_pre(const mhc_bf16* partials, int num_partials, int64_t partial_stride,
                                 const mhc_bf16* residual, const float* post, const float* comb, const float* pre,
                                 const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
                                 mhc_bf16* residual_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
                                 float* post_out, float* comb_out, float* pre_out, int rows, int hidden,
                                 int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (num_partials < 1 || num_partials > kMaxPartials) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!partials || !aligned(partials, 16) || partial_stride % 8 != 0) return MHC_ERR_INVALID_ARG;
  if (num_partials > 1 && partial_stride == 0) return MHC_ERR_INVALID_ARG;
  mhc_status st = check_mixes(residual, post, comb, residual_out);
  if (st != MHC_OK) return st;
  Params p{};
  p.partials = reinterpret_cast<const __nv_bfloat16*>(partials);
  p.pstride = partial_stride;
  p.P = num_partials;
  p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  p.post = post;
  p.comb = comb;
  p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
  p.write_res = 1;
  p.R = rows;
  p.H = hidden;
  st = fill_tail(p, pre, norm_weight, norm_eps, coeffs, layer_input, mxfp8, post_out, comb_out, pre_out, rows,
                 hidden, hc_mult, workspace, ws_bytes);
  if (st != MHC_OK) return st;
  return dispatch_n<kPartials>(p, hc_mult, stream);
}

mhc_status mhc_boundary_moe_finalize(const mhc_bf16* gemm2_permuted, int num_permuted, const float* expert_weights,
                                     const int32_t* expanded_idx_to_permuted_idx, int top_k,
                                     const mhc_bf16* shared_output, const mhc_bf16* residual, const float* post,
                                     const float* comb, const float* pre, const mhc_bf16* norm_weight,
                                     float norm_eps, const mhc_coeff_args* coeffs, mhc_bf16* residual_out,
                                     mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8, float* post_out,
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
                                      mhc_bf16* residual_out, int rows, int hidden, int hc_mult,
                                      mhc_stream stream) {
  if (!shape_ok(rows, hidden, hc_mult)) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (num_partials < 1 || num_partials > kMaxPartials) return MHC_ERR_UNSUPPORTED_SHAPE;
  if (!partials || !aligned(partials, 16) || partial_stride % 8 != 0) return MHC_ERR_INVALID_ARG;
  if (num_partials > 1 && partial_stride == 0) return MHC_ERR_INVALID_ARG;
  mhc_status st = check_mixes(residual, post, comb, residual_out);
  if (st != MHC_OK) return st;
  Params p{};
  p.partials = reinterpret_cast<const __nv_bfloat16*>(partials);
  p.pstride = partial_stride;
  p.P = num_partials;
  p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  p.post = post;
  p.comb = comb;
  p.residual_out = reinterpret_cast<__nv_bfloat16*>(residual_out);
  p.write_res = 1;
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
  const int blocks = static_cast<int>((lanes + 255) / 256);
  mxfp8_rows_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(x), rows, hidden, out->data,
                                                 out->scale, out->swizzled_128x4 != 0);
  if (cudaGetLastError() != cudaSuccess) return MHC_ERR_CUDA;
  if (out->swizzled_128x4) {
    const int scols = hidden / 32;
    const int rows_p = (rows + 127) / 128 * 128;
    const int cols_p = (scols + 3) / 4 * 4;
    if (rows_p != rows || cols_p != scols) {
      const int total = rows_p * cols_p;
      scale_padding_kernel<<<(total + 255) / 256 < 1024 ? (total + 255) / 256 : 1024, 256, 0, stream>>>(
          out->scale, rows, hidden);
      if (cudaGetLastError() != cudaSuccess) return MHC_ERR_CUDA;
    }
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

int64_t mhc_debug_set_wait(int64_t budget_ns, int extra_arrivals) {
  const int64_t old = g_budget_ns;
  if (budget_ns > 0) g_budget_ns = budget_ns;
  g_extra_arrivals = extra_arrivals < 0 ? 0 : extra_arrivals;
  return old;
}

}  // extern "C"
