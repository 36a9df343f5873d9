"""Per-phase clock stamps of the two-kernel boundary, for measurement only.

`build_stamped()` compiles a copy of the library whose streaming and tail
kernels record the GPU's global timer (%globaltimer, ns) at their phase
boundaries: thread 0 of every block, into a device ring of the last 8 launches
of each block. The product library is not touched; the copy is built into a
temporary directory. `summary()` turns one ring into the phase table (ns after
the streaming kernel's first wait return of the same boundary, latest block
unless marked median), averaged as medians over the boundaries in the ring.

Streaming kernel events: 0 start, 1 before the wait, 2 after the wait, 3 mixes
staged, 7 tensor-map copies of the rows landed (staged form), 6 first row data
in (block's warp 0), 4 all row pairs done, 5 end.
Tail events: 0 start, 4 at the wait (layer blocks), 1 after the wait, 3 first
layer task's data in (layer blocks) or records added up (coefficient blocks),
4/5 Sinkhorn start / end (coefficient blocks), 6 end; word 7 holds the block
kind (1 layer input, 2 coefficients).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

from . import build

_PRE = r'''
namespace mhc {
__device__ unsigned long long g_ts[8][160][8];   // streaming kernel [slot][block][event]
__device__ unsigned long long g_tt[8][320][8];   // tail kernel
__device__ unsigned g_seq_s[160], g_seq_t[320];  // launches seen by each block
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
}
'''

_POST = r'''
extern "C" __attribute__((visibility("default"))) int mhc_phase_read(void* s, size_t sb, void* t, size_t tb) {
  return (cudaMemcpyFromSymbol(s, mhc::g_ts, sb) == cudaSuccess &&
          cudaMemcpyFromSymbol(t, mhc::g_tt, tb) == cudaSuccess) ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int mhc_phase_reset(void) {
  static unsigned zero[320];
  static unsigned long long zs[8 * 320 * 8];
  return (cudaMemcpyToSymbol(mhc::g_seq_s, zero, sizeof(unsigned) * 160) == cudaSuccess &&
          cudaMemcpyToSymbol(mhc::g_seq_t, zero, sizeof(unsigned) * 320) == cudaSuccess &&
          cudaMemcpyToSymbol(mhc::g_ts, zs, sizeof(unsigned long long) * 8 * 160 * 8) == cudaSuccess &&
          cudaMemcpyToSymbol(mhc::g_tt, zs, sizeof(unsigned long long) * 8 * 320 * 8) == cudaSuccess) ? 0 : 1;
}
'''

# (anchor, code, insert after the anchor?)
_STAMPS = [
    ("  const int npairs = (R + 1) >> 1;\n",
     "  unsigned tslot = 0;\n  const unsigned long long t0s = mhc::gtimer();\n"
     "  if (tid == 0) {\n    tslot = atomicAdd(&mhc::g_seq_s[blockIdx.x], 1u) & 7u;\n"
     "    mhc::g_ts[tslot][blockIdx.x][0] = t0s;\n  }\n", True),
    ("  griddep_wait();\n  griddep_launch_dependents();\n  PairLoads<N> cur;",
     "  if (tid == 0) mhc::g_ts[tslot][blockIdx.x][1] = mhc::gtimer();\n", False),
    ("  griddep_wait();\n  griddep_launch_dependents();\n  PairLoads<N> cur;",
     "  if (tid == 0) mhc::g_ts[tslot][blockIdx.x][2] = mhc::gtimer();\n", True),
    ("  if (FRONT == kMoe && warp < npairs) load_pair<N, FRONT>(p, warp * 2 + rq, h0, e2p_s, cur);\n",
     "  if (tid == 0) mhc::g_ts[tslot][blockIdx.x][3] = mhc::gtimer();\n", True),
    ("        for (int j = 0; j < N; ++j) unpack4x2(cur.rv[j], rf[j]);\n",
     "        if (tid == 0 && q == warp) mhc::g_ts[tslot][blockIdx.x][6] = mhc::gtimer() + (rf[0][0].x == 12345.f);\n",
     True),
    ("  const int mtiles = (R + 15) >> 4;\n", "  if (tid == 0) mhc::g_ts[tslot][blockIdx.x][4] = mhc::gtimer();\n", False),
    ("        if (col + 1 < C) dst[1] = (acc[0][2 * h + 1] + acc[1][2 * h + 1]) + acc[2][2 * h + 1];\n      }\n    }\n  }\n",
     "  __syncthreads();\n  if (tid == 0) mhc::g_ts[tslot][blockIdx.x][5] = mhc::gtimer();\n", True),
    ("  const int bid = blockIdx.x;\n  const int lbid = p.tail_coeff_first ? bid - p.tail_coeff_blocks : bid;\n",
     "  unsigned tslot = 0;\n  const unsigned long long t0t = mhc::gtimer();\n"
     "  if (tid == 0) {\n    tslot = atomicAdd(&mhc::g_seq_t[bid], 1u) & 7u;\n    mhc::g_tt[tslot][bid][0] = t0t;\n"
     "    mhc::g_tt[tslot][bid][7] = (lbid >= 0 && lbid < p.tail_layer_blocks) ? 1 : 2;\n  }\n", True),
    ("    griddep_wait();\n    griddep_launch_dependents();\n    if (w0 < T) layer_load",
     "    if (tid == 0) mhc::g_tt[tslot][bid][4] = mhc::gtimer();\n", False),
    ("    griddep_wait();\n    griddep_launch_dependents();\n"
     "    if (w0 < T) layer_load<N>(p, w0 / GT, (w0 % GT) * 4 + rq, lane, false, cur);\n",
     "    if (tid == 0) mhc::g_tt[tslot][bid][1] = mhc::gtimer();\n", True),
    ("      const float inv = rsqrtf(__fdiv_rn(a, static_cast<float>(H)) + p.norm_eps);\n      if (g < G) {",
     "      if (tid == 0 && t == w0) mhc::g_tt[tslot][bid][3] = mhc::gtimer();\n", False),
    ("    griddep_wait();\n    griddep_launch_dependents();\n    constexpr int V4 = RED / 4;\n",
     "    if (tid == 0) mhc::g_tt[tslot][bid][1] = mhc::gtimer();\n", True),
    ("      // warp s < nk: the comb (Sinkhorn) of row s of the batch; the pre and post of",
     "      if (tid == 0 && k0 == 0) mhc::g_tt[tslot][bid][3] = mhc::gtimer();\n", False),
    ("            sinkhorn_iterate<N>(M, p.iters, p.sk_eps);\n",
     "            if (tid == 0 && k0 == 0) mhc::g_tt[tslot][bid][4] = mhc::gtimer();\n", False),
    ("            sinkhorn_iterate<N>(M, p.iters, p.sk_eps);\n",
     "            if (tid == 0 && k0 == 0) mhc::g_tt[tslot][bid][5] = mhc::gtimer();\n", True),
    ("      __syncthreads();  // the slots are refilled by the next batch\n    }\n  }\n",
     "  __syncthreads();\n  if (tid == 0) mhc::g_tt[tslot][bid][6] = mhc::gtimer();\n", True),
]


# stamps of code that only some forms of the kernel have: inserted where found
_OPTIONAL = [
    ("    if (!mbar_wait_bounded(sbar, 0, deadline)) record_error(status, MHC_ERR_DEVICE_TIMEOUT);\n",
     "    if (tid == 0) mhc::g_ts[tslot][blockIdx.x][7] = mhc::gtimer();\n", True),
]


def instrument(src: str) -> str:
    """The kernel source with the stamps inserted (each anchor must occur once)."""
    head = "namespace mhc {\n\nconstexpr int kCols"
    if src.count(head) != 1:
        raise RuntimeError("kernel source layout changed: namespace anchor")
    src = src.replace(head, _PRE + "\n" + head, 1)
    for anchor, code, after in _OPTIONAL:
        if src.count(anchor) == 1:
            i = src.index(anchor) + (len(anchor) if after else 0)
            src = src[:i] + code + src[i:]
    for anchor, code, after in _STAMPS:
        if src.count(anchor) != 1:
            raise RuntimeError(f"kernel source layout changed: {anchor[:60]!r}")
        i = src.index(anchor)
        j = i + len(anchor) if after else i
        src = src[:j] + code + src[j:]
    return src + _POST


def build_stamped(out_dir: str | None = None) -> str:
    """Compile the stamped copy of the library; return the path of its .so."""
    out_dir = out_dir or tempfile.mkdtemp(prefix="mhc_stamped_")
    os.makedirs(out_dir, exist_ok=True)
    with open(build.SOURCES[0]) as f:
        src = instrument(f.read())
    src = src.replace('#include "mhc_device.cuh"', '#include "%s"' % os.path.join(build.CSRC, "mhc_device.cuh"))
    src = src.replace('#include "../../include/mhc.h"', '#include "%s"' % os.path.join(build.INCLUDE, "mhc.h"))
    cu = os.path.join(out_dir, "mhc_boundary_stamped.cu")
    with open(cu, "w") as f:
        f.write(src)
    lib = os.path.join(out_dir, "libmhc.so")
    res = subprocess.run([build._nvcc(), *build.NVCC_FLAGS, "-I", build.INCLUDE, "-o", lib, cu],
                         capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr}")
    return lib


def reset(L: ctypes.CDLL):
    L.mhc_phase_reset.restype = ctypes.c_int
    if L.mhc_phase_reset() != 0:
        raise RuntimeError("mhc_phase_reset failed")


def read(L: ctypes.CDLL):
    S = np.zeros((8, 160, 8), dtype=np.uint64)
    T = np.zeros((8, 320, 8), dtype=np.uint64)
    L.mhc_phase_read.restype = ctypes.c_int
    L.mhc_phase_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t]
    if L.mhc_phase_read(S.ctypes.data, S.nbytes, T.ctypes.data, T.nbytes) != 0:
        raise RuntimeError("mhc_phase_read failed")
    return S, T


PHASES = [  # key, what
    ("prewait", "streaming: last block reaches its wait"),
    ("staged_med", "streaming: tensor-map copies of the rows landed (median block; staged form only)"),
    ("mixes_med", "streaming: mixes staged (median block)"),
    ("data_med", "streaming: first rows' data in (median block)"),
    ("rows", "streaming: all row pairs post-mixed"),
    ("stream_end", "streaming: last block ends (projection done)"),
    ("tail_wait", "tail: first wait return"),
    ("records", "tail: rows' records added up (coefficient blocks)"),
    ("sk_start", "tail: Sinkhorn starts"),
    ("sk_end", "tail: Sinkhorn ends"),
    ("layer_data", "tail: first layer task's data in (layer blocks)"),
    ("layer_end", "tail: layer-input blocks end"),
    ("tail_end", "tail: last block ends"),
    ("next_wait", "next boundary: streaming kernel's first wait return"),
]


def summary(S: np.ndarray, T: np.ndarray, G: int) -> dict:
    """Medians over the boundaries in the ring of each phase's time, ns after the
    streaming kernel's first wait return."""
    nt = int((T[0, :, 7] != 0).sum())
    out = {k: [] for k, _ in PHASES}
    for s in range(8):
        st = S[s, :G].astype(np.int64)
        tt = T[s, :nt].astype(np.int64)
        if nt == 0 or (st[:, 2] == 0).any() or (tt[:, 1] == 0).any() or (st[:, 5] == 0).any():
            continue
        base = st[:, 2].min()
        out["prewait"].append(st[:, 1].max() - base)
        out["mixes_med"].append(int(np.median(st[:, 3])) - base)
        if (st[:, 7] != 0).all():
            out["staged_med"].append(int(np.median(st[:, 7])) - base)
        out["data_med"].append(int(np.median(st[:, 6])) - base)
        out["rows"].append(st[:, 4].max() - base)
        out["stream_end"].append(st[:, 5].max() - base)
        out["tail_wait"].append(tt[:, 1].min() - base)
        coef, lay = tt[tt[:, 7] == 2], tt[tt[:, 7] == 1]
        if len(coef):
            out["records"].append(coef[:, 3].max() - base)
            out["sk_start"].append(coef[:, 4].max() - base)
            out["sk_end"].append(coef[:, 5].max() - base)
        if len(lay):
            out["layer_data"].append(lay[:, 3].max() - base)
            out["layer_end"].append(lay[:, 6].max() - base)
        out["tail_end"].append(tt[:, 6].max() - base)
        nxt = S[(s + 1) % 8, :G].astype(np.int64)
        if (nxt[:, 2] != 0).all() and nxt[:, 2].min() > tt[:, 6].max():
            out["next_wait"].append(nxt[:, 2].min() - base)
    return {k: (int(np.median(v)) if v else None) for k, v in out.items()}
