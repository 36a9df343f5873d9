/*
 * mhc.h - C ABI of the B200 (sm_100a) mHC decode boundary library, libmhc.so.
 *
 * The boundary sits between two decoder sublayers of a DeepSeek-V4-style decode
 * step. It reduces the previous sublayer's output into the hc_mult residual
 * streams (mHC post), collapses and RMS-normalises the streams into the next
 * sublayer's input (mHC pre), optionally as MXFP8, and computes the next mHC
 * coefficients. Sources, by page title and section:
 *   [boundary]   vllm ...specialized_decode.boundary.boundary:
 *                Boundaries.first / sublayer / post_only / _pre / _reduce,
 *                BoundaryState, empty_quantized_layer_input
 *   [all_reduce] vllm ...specialized_decode.boundary.all_reduce:
 *                BoundaryAllReduce.__call__ / finalize
 *   [decode]     vllm ...specialized_decode.runtime.decode:
 *                SpecializedDecode.run (the layer loop), _head
 *
 * Notation: R = rows (decode tokens), H = hidden, n = hc_mult, K = n*H,
 * C = 2n + n^2 (coefficient logits), P = partial buffers, k = top_k.
 *
 * Conventions shared by every entry point
 *   - bf16 tensors are passed as mhc_bf16 (the raw 16-bit pattern), fp32 as
 *     float, all row-major and contiguous unless a stride is given.
 *   - Every pointer is a DEVICE pointer owned by the caller. The library never
 *     allocates, frees or keeps a pointer after the call returns.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream) and
 *     do not synchronise the host. Host-side argument checks happen before any
 *     launch; a call that returns an error launched nothing.
 *   - Kernels are launched with programmatic stream serialization (dependent
 *     launch): a boundary kernel may start while the kernel before it on the
 *     stream is finishing, and reads the weights (fn, scale, base, norm_weight)
 *     before waiting for that kernel. So weights must not be written by the
 *     kernel launched immediately before on the same stream if that kernel
 *     triggers dependent launches (no kernel of this library writes weights;
 *     kernels that do not trigger, like ordinary library kernels, are waited
 *     for in full). Activations are read only after the wait.
 *   - Errors are returned, never raised or aborted on. Errors found by a kernel
 *     (a wait that ran out, a gather index out of range) are recorded in the
 *     workspace and read with mhc_get_device_status.
 *   - Shapes: 1 <= R <= 128, H a multiple of 64 with H/64 <= 148 (H <= 9472),
 *     n in {1, 2, 4}, 1 <= P <= 16, 1 <= k <= 16.
 *   - Alignment: bf16 tensors and fn 16-byte aligned, MXFP8 data 8-byte aligned,
 *     fp32 vectors 4-byte aligned; partial_stride a multiple of 8 elements.
 *   - residual_out may be the same buffer as residual (in place) but must not
 *     partially overlap it. No other output may overlap any input.
 */
#ifndef MHC_H
#define MHC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MHC_API __attribute__((visibility("default")))
#else
#define MHC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mhc_bf16;         /* bfloat16 bit pattern */
typedef struct CUstream_st* mhc_stream; /* the same type as cudaStream_t */

typedef enum {
  MHC_OK = 0,
  MHC_ERR_INVALID_ARG = 1,       /* NULL where required, bad alignment, eps < 0 ... */
  MHC_ERR_UNSUPPORTED_SHAPE = 2, /* rows/hidden/hc_mult/P/top_k outside the limits */
  MHC_ERR_WORKSPACE = 3,         /* workspace NULL, misaligned or too small */
  MHC_ERR_CUDA = 4,              /* a CUDA runtime call failed (launch, query) */
  MHC_ERR_DEVICE_TIMEOUT = 5,    /* device: a bounded wait gave up */
  MHC_ERR_DEVICE_INDEX = 6       /* device: expanded_idx_to_permuted_idx past the end */
} mhc_status;

/* Weights and scalars of the next-coefficient step, as the stock mHC pre takes
 * them ([boundary] Boundaries.sublayer passes fn, scale, base, rms_norm_eps,
 * hc_eps, hc_eps, hc_post_alpha, hc_sinkhorn_iters).
 *   fn    [n*H, C] fp32; row k = j*H + h is stream j, column h of a row's streams.
 *         Columns: [pre 0..n-1 | post n..2n-1 | comb 2n..], comb column
 *         2n + j*n + i is comb[j][i] (stream j into stream i).
 *   scale [3] fp32, one per group pre / post / comb.
 *   base  [C] fp32.
 * Per row r, with v the row's streams flattened to K values:
 *   inv  = 1/sqrt(mean(v^2) + rms_eps);  l_c = scale[group c] * inv * (v . fn[:,c]) + base[c]
 *   pre  = sigmoid(l_pre) + pre_eps;     post = post_alpha * sigmoid(l_post)
 *   comb = Sinkhorn(l_comb, sinkhorn_iters, sinkhorn_eps):
 *          M = exp(L - max L); repeat: rows /= (row sum + eps), then columns /= (column sum + eps).
 *   fn_packed  optional: fn as mhc_projection_pack wrote it. When set, the
 *         boundary reads it instead of fn (fn may then be NULL) and gives
 *         bitwise the same results; it spares the kernel the split of fn into
 *         bf16 terms at every call, at 1.55x the bytes of fn for n = 4.
 * Constraints: fn or fn_packed set, eps values >= 0, 0 <= sinkhorn_iters <= 1000.
 * Supported spread of the comb logits: the kernel takes M in fp32, so a comb
 * logit more than about 87 below the largest one of its row's n*n gives a
 * subnormal or zero entry of M where the exact definition keeps a tiny positive
 * weight. Logits within 80 of the largest are tested against the exact
 * definition; wider spreads are out of contract. */
typedef struct {
  const float* fn;
  const float* scale;
  const float* base;
  float rms_eps;
  float pre_eps;
  float sinkhorn_eps;
  float post_alpha;
  int sinkhorn_iters;
  const void* fn_packed;
} mhc_coeff_args;

/* MXFP8 layer input ([boundary] empty_quantized_layer_input: E4M3 data [R, H] and
 * a uint8 scale buffer in FlashInfer's swizzled 128x4 layout).
 *   data  [R, H] E4M3 bytes (OCP "fn" variant), RNE, saturating to +-448.
 *   scale E8M0 bytes, one per 32 consecutive elements of a row, e = the smallest
 *         integer with amax <= 448 * 2^e (clamped to [-127, 127]), byte e + 127.
 *         swizzled_128x4 != 0: mhc_mxfp8_scale_bytes(R, H, 1) bytes; the [R, H/32]
 *         scale matrix padded to 128-row x 4-column tiles of 512 bytes, tiles in
 *         row-major order, (r, c) inside a tile at (r%32)*16 + (r/32)*4 + c;
 *         padding bytes are written as 0.
 *         swizzled_128x4 == 0: linear [R, H/32].
 *   A block holding NaN or Inf is out of contract: scale 0xFF, data 0x7F. */
typedef struct {
  uint8_t* data;
  uint8_t* scale;
  int swizzled_128x4;
} mhc_mxfp8_out;

/* Bytes of workspace the boundary entry points need for (rows, hidden, hc_mult):
 * a 1 KB header (the status word kernels record errors in) and the per-block
 * partial sums that the tail of a boundary adds up. A workspace sized for R rows
 * serves every call with rows <= R and the same hidden and hc_mult. It must be
 * 256-byte aligned, zeroed once before first use (mhc_workspace_init; the
 * partial sums are rewritten by every call) and used by one stream at a time:
 * calls sharing a workspace must not overlap on the GPU. Returns 0 for
 * unsupported shapes. */
MHC_API size_t mhc_workspace_bytes(int rows, int hidden, int hc_mult);

/* Bytes of the MXFP8 scale buffer: roundup(R,128) * roundup(H/32, 4) when
 * swizzled, R * H/32 when linear. Returns 0 for H not a multiple of 32. */
MHC_API size_t mhc_mxfp8_scale_bytes(int rows, int hidden, int swizzled_128x4);

/* Zero the workspace on `stream` (cudaMemsetAsync). Needed once before first use. */
MHC_API mhc_status mhc_workspace_init(void* workspace, size_t ws_bytes, mhc_stream stream);

/* fn [n*H, C] fp32 rewritten once, at weight-load time, into the form the
 * projection's tensor-core tiles read (no counterpart in the method: a layout
 * of the same weights). Each value f becomes three bf16 terms hi + mid + lo
 * equal to f to 2^-24 (hi = bf16(f), mid = bf16(f - hi), lo = bf16(f - hi - mid)),
 * grouped per 64-column block of H as [3][CP8][n*64 + 8] with CP8 = C rounded
 * up to 8 and zeros in the padding. The layout is private to this library
 * version: pass the result only as mhc_coeff_args.fn_packed.
 *   mhc_projection_pack_bytes: H/64 * 3 * CP8 * (n*64 + 8) * 2 bytes, 0 for an
 *     unsupported (hidden, hc_mult).
 *   mhc_projection_pack: fn 4-byte aligned, packed 16-byte aligned and
 *     mhc_projection_pack_bytes long; asynchronous on stream, an ordinary
 *     launch (a boundary launched after it on the stream sees the result). */
MHC_API size_t mhc_projection_pack_bytes(int hidden, int hc_mult);
MHC_API mhc_status mhc_projection_pack(const float* fn, void* packed, int hidden, int hc_mult, mhc_stream stream);

/* Full boundary after a sublayer with TP-partial output ([all_reduce]
 * BoundaryAllReduce.__call__, [boundary] Boundaries.sublayer / _reduce):
 *   x[r,h]        = sum_p partials[p*partial_stride + r*H + h]      (fp32)
 *   new[r,i,h]    = bf16( sum_j comb[r,j,i]*residual[r,j,h] + post[r,i]*x[r,h] )
 *   residual_out  = new                                              [R, n, H]
 * and when pre != NULL (pre is the pre-mix carried from the previous boundary,
 * [boundary] BoundaryState.pre):
 *   c[r,h]        = sum_j pre[r,j]*new[r,j,h]
 *   layer_input   = bf16( c * rsqrt(mean_h c^2 + norm_eps) * norm_weight[h] )  [R, H]
 *   mxfp8 (optional, may be NULL) = MXFP8 of layer_input
 *   coeffs (optional, may be NULL) -> post_out [R,n], comb_out [R,n,n], pre_out [R,n]
 *     computed from the new streams (see mhc_coeff_args).
 * pre == NULL is the residual-only variant ([boundary] Boundaries._reduce with no
 * pre and no norm): then norm_weight, layer_input, mxfp8 and coeffs must be NULL.
 * aux_out (optional, may be NULL; 16-byte aligned) receives the hidden state a
 * capturing layer keeps ([boundary] Boundaries.sublayer with capture_aux, and
 * [decode] SpecializedDecode.run after the last layer): the mean of the new
 * streams, aux[r,h] = bf16( (sum_j new[r,j,h]) / n ), summed in stream order in
 * fp32 and rounded once.  [R, H]
 * The decode step's final head ([decode] SpecializedDecode._head:
 * norm(hc_collapse(streams, pre))) is this call with the carried pre, the final
 * norm's weight and coeffs = NULL: layer_input is then the step's hidden state.
 * Inputs post [R,n], comb [R,n,n], pre [R,n] are fp32; norm_weight [H] bf16.
 * workspace: see mhc_workspace_bytes. */
MHC_API mhc_status mhc_boundary_post_pre(
    const mhc_bf16* partials, int num_partials, int64_t partial_stride,
    const mhc_bf16* residual, const float* post, const float* comb, const float* pre,
    const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
    mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
    float* post_out, float* comb_out, float* pre_out,
    int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream);

/* mhc_boundary_post_pre with the partials given as a table: partials is a HOST
 * array of num_partials DEVICE pointers, each to a [R, H] bf16 partial (16-byte
 * aligned). A pointer may be another GPU's memory (peer access or
 * mhc_ipc_import): this is the tensor-parallel boundary, where every rank's
 * kernel sums all ranks' partials itself with plain peer loads, in pointer
 * order, instead of an all-reduce before it ([boundary] Boundaries.post_only:
 * tensor_model_parallel_all_reduce then mhc_post; [all_reduce]
 * BoundaryAllReduce.__call__). The table is read during the call only. The
 * caller orders the accesses: every partial complete before the call (e.g. a
 * barrier across the ranks after their sublayers) and no partial overwritten
 * until every rank's boundary has read it. pre == NULL is the residual-only
 * form, which needs no workspace. */
MHC_API mhc_status mhc_boundary_post_pre_ptrs(
    const mhc_bf16* const* partials, int num_partials,
    const mhc_bf16* residual, const float* post, const float* comb, const float* pre,
    const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
    mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
    float* post_out, float* comb_out, float* pre_out,
    int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream);

/* Publish/collect mailbox of a tensor-parallel group, without multicast
 * ([all_reduce] BoundaryAllReduce.publish_target / mark_published: a producer
 * stores its bf16 contribution, negative zero cleared, into slot [rank][token]
 * of the mailbox; the consumer's reduction waits for it. Here each rank's
 * mailbox is its own device memory and producers store into every rank's
 * mailbox, over NVLink for the peers'.)
 * Layout of a mailbox (mhc_mailbox_bytes(W, M, H) bytes, 256-byte aligned, M
 * the row capacity): a 256-byte header (status word at byte 0; at bytes 8 and
 * 12 the round + 1 last consumed for each parity), then slots bf16
 * [2][W][M][H]. A slot element holding negative zero (0x8000) is "not yet
 * written": producers never store it, the consumer writes it back into every
 * element it has read. Round t uses parity t & 1, so a producer may run one
 * round ahead of a consumer.
 *   mhc_mailbox_bytes: 0 for world outside [1, 16] or an unsupported (M, H).
 *   mhc_mailbox_init: header zero, every slot element negative zero (a kernel
 *     on `stream`; bytes = mhc_mailbox_bytes(...), a multiple of 16).
 *   mhc_mailbox_publish: producer `rank` of a group of `world` stores x
 *     [rows, H] bf16 (16-byte aligned, rows <= M) into slot [t & 1][rank] of
 *     every consumer's mailbox (mailboxes: HOST array of `world` device
 *     pointers, this GPU's or peers' via mhc_ipc_import), with each negative
 *     zero stored as positive zero. Before writing into a consumer's mailbox it
 *     waits (bounded, mhc_debug_set_wait) until that consumer has consumed
 *     round t - 2; on timeout it writes nothing there and records
 *     MHC_ERR_DEVICE_TIMEOUT in its OWN mailbox's status word (read it with
 *     mhc_get_device_status(mailboxes[rank])).
 *   mhc_boundary_collect: the consumer's boundary of round t over `rows`
 *     (<= M) tokens: as mhc_boundary_post_pre with the W slots of parity t & 1
 *     as the partials (summed in producer order). Its streaming kernel re-reads
 *     each slot element until it is not negative zero (bounded; a timeout
 *     records MHC_ERR_DEVICE_TIMEOUT in the workspace, which is required, also
 *     for the residual-only form) and marks it negative zero again once read.
 *     A one-thread kernel then marks round t consumed. round must be below
 *     0xffffffff.
 * Producers and consumers on different GPUs run concurrently; the waits are
 * the only ordering between them. A published value of negative zero arrives
 * as positive zero (the sum then differs at most in the sign of a zero). */
MHC_API size_t mhc_mailbox_bytes(int world, int max_rows, int hidden);
MHC_API mhc_status mhc_mailbox_init(void* mailbox, size_t bytes, mhc_stream stream);
MHC_API mhc_status mhc_mailbox_publish(const mhc_bf16* x, int rows, int hidden, int rank, uint32_t round,
                                       void* const* mailboxes, int world, int max_rows, mhc_stream stream);
MHC_API mhc_status mhc_boundary_collect(
    void* mailbox, int world, int max_rows, uint32_t round,
    const mhc_bf16* residual, const float* post, const float* comb, const float* pre,
    const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
    mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
    float* post_out, float* comb_out, float* pre_out,
    int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream);

/* Device memory shared between processes (one process per GPU), for the
 * partial table above (no counterpart on the pages, which use a multicast
 * mailbox; nothing here uses multicast).
 *   mhc_ipc_handle_bytes: size of a handle (a CUDA IPC handle of the
 *     allocation holding the pointer, plus the pointer's offset into it).
 *   mhc_ipc_export: write the handle of dev_ptr (device memory from cudaMalloc
 *     or a caching allocator built on it) into handle_out.
 *   mhc_ipc_import: map a handle exported by ANOTHER process; *dev_ptr_out is
 *     the same byte the exporter's pointer names. Opening a handle of the
 *     calling process fails (MHC_ERR_CUDA).
 *   mhc_ipc_release: unmap a pointer from mhc_ipc_import.
 * The exporter must keep the memory allocated until every importer released it. */
MHC_API size_t mhc_ipc_handle_bytes(void);
MHC_API mhc_status mhc_ipc_export(const void* dev_ptr, void* handle_out);
MHC_API mhc_status mhc_ipc_import(const void* handle, void** dev_ptr_out);
MHC_API mhc_status mhc_ipc_release(void* dev_ptr);

/* Boundary after a MoE sublayer whose output was left unfinalized ([all_reduce]
 * BoundaryAllReduce.finalize, [boundary] Boundaries._reduce):
 *   x[r,h] = shared_output[r,h] + sum_t expert_weights[r*top_k+t] *
 *            gemm2_permuted[e2p[r*top_k+t]*H + h]
 * with e2p = expanded_idx_to_permuted_idx [R*top_k] int32: an entry < 0 adds
 * nothing; an entry >= num_permuted adds nothing and records
 * MHC_ERR_DEVICE_INDEX. gemm2_permuted [num_permuted, H] bf16, expert_weights
 * [R, top_k] fp32, shared_output [R, H] bf16. Everything after x is as in
 * mhc_boundary_post_pre, including the residual-only variant (pre == NULL). */
MHC_API mhc_status mhc_boundary_moe_finalize(
    const mhc_bf16* gemm2_permuted, int num_permuted, const float* expert_weights,
    const int32_t* expanded_idx_to_permuted_idx, int top_k, const mhc_bf16* shared_output,
    const mhc_bf16* residual, const float* post, const float* comb, const float* pre,
    const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
    mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
    float* post_out, float* comb_out, float* pre_out,
    int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream);

/* Residual-only boundary ([boundary] Boundaries.post_only: all-reduce then mHC
 * post, streams only): residual_out = bf16(comb-mix of residual + post * sum of
 * partials), and aux_out (may be NULL) as in mhc_boundary_post_pre. Needs no
 * workspace. */
MHC_API mhc_status mhc_boundary_residual_only(
    const mhc_bf16* partials, int num_partials, int64_t partial_stride,
    const mhc_bf16* residual, const float* post, const float* comb,
    mhc_bf16* residual_out, mhc_bf16* aux_out, int rows, int hidden, int hc_mult, mhc_stream stream);

/* The stock mHC pre without a reduction ([boundary] Boundaries._pre), two forms:
 *   residual != NULL, x == NULL: coefficients of the given streams [R, n, H]; with
 *     layer_input != NULL also the layer input from pre_mix [R, n] (required then).
 *   x != NULL, residual == NULL: the first layer ([boundary] Boundaries.first). The
 *     embedding x [R, H] is broadcast to the n streams; the identity pre-mix
 *     selects stream 0, so layer_input = bf16(x * rsqrt(mean x^2 + norm_eps) * w).
 *     pre_mix must be NULL. residual_out (may be NULL) receives the broadcast
 *     streams [R, n, H]. The coefficients are those of the broadcast streams with
 *     fn [n*H, C] (the first layer's hc_attn_fn_broadcast).
 * post_out, comb_out and pre_out are always written. */
MHC_API mhc_status mhc_coeffs(
    const mhc_bf16* residual, const mhc_coeff_args* coeffs, const float* pre_mix,
    const mhc_bf16* x, mhc_bf16* residual_out,
    const mhc_bf16* norm_weight, float norm_eps, mhc_bf16* layer_input,
    float* post_out, float* comb_out, float* pre_out,
    int rows, int hidden, int hc_mult, void* workspace, size_t ws_bytes, mhc_stream stream);

/* MXFP8 of a bf16 [R, H] matrix (x, row-major, 16-byte aligned), same encoding
 * and scale layouts as mhc_mxfp8_out. 1 <= R <= 65535, H a multiple of 32. */
MHC_API mhc_status mxfp8_quantize_rows(const mhc_bf16* x, int rows, int hidden,
                               const mhc_mxfp8_out* out, mhc_stream stream);

/* mhc_boundary_post_pre for callers that cannot allocate device memory.
 * The pages have no counterpart: this entry point exists for callers such as a
 * plugin hosted by a runtime that owns all device memory (it is only handed
 * tensors), code running while a CUDA graph is captured (cudaMalloc is not a
 * stream operation), or a serving loop that must not take the allocator's locks.
 * Arguments and results are those of mhc_boundary_post_pre without the
 * workspace: the scratch is a fixed device array inside the library, 1,893,376
 * bytes (the workspace of rows 128, hidden 7168, hc_mult 4), which every GPU
 * that loads the library holds until the process exits. Limits: rows <= 128,
 * hidden <= 7168, hc_mult <= 4; larger shapes return MHC_ERR_WORKSPACE.
 * The first call on a device looks up the array's device address (one
 * cudaGetSymbolAddress per device and CUDA context, with that device current;
 * after a device reset the new context's address is looked up again); make that
 * first call before any stream capture. Every call on a device shares the array:
 * calls that overlap on the GPU (other streams, other threads) race on it and
 * must be serialised by the caller. A kernel-side error (a wait that ran out) is
 * recorded in the array and not reported; use mhc_boundary_post_pre with a
 * workspace to read it. Allocates nothing. */
MHC_API mhc_status mhc_boundary_post_pre_noalloc(
    const mhc_bf16* partials, int num_partials, int64_t partial_stride,
    const mhc_bf16* residual, const float* post, const float* comb, const float* pre,
    const mhc_bf16* norm_weight, float norm_eps, const mhc_coeff_args* coeffs,
    mhc_bf16* residual_out, mhc_bf16* aux_out, mhc_bf16* layer_input, const mhc_mxfp8_out* mxfp8,
    float* post_out, float* comb_out, float* pre_out,
    int rows, int hidden, int hc_mult, mhc_stream stream);

/* Wait for `stream`, then read and clear the error a kernel recorded in
 * `workspace` (MHC_OK when none). The only entry point that synchronises. */
MHC_API mhc_status mhc_get_device_status(void* workspace, mhc_stream stream);

/* Static, human-readable name of a status code. */
MHC_API const char* mhc_status_string(mhc_status status);

/* Test hook for the bounded waits. A kernel waits on the TMA copies of its fn
 * slice (and the mailbox kernels on their slots and consumed words) with a time limit: `budget_ns`
 * > 0 sets it (default 1e9 ns, counted as
 * 2 SM cycles per ns); `extra_units` makes that wait expect that many 16-byte
 * units more than are copied, so that it can never complete and runs out
 * (recording MHC_ERR_DEVICE_TIMEOUT). Affects launches made after the call by
 * this process. Returns the previous budget. */
MHC_API int64_t mhc_debug_set_wait(int64_t budget_ns, int extra_units);

#ifdef __cplusplus
}
#endif

#endif /* MHC_H */
