/*
 * bb_attn.h -- C ABI of libbbattn.so: BigBird ITC block-sparse attention,
 * forward and backward, on NVIDIA B200 (sm_100a).
 *
 * The operation (web page "models 仓库中的 BigBird：线性复杂度稀疏注意力与长序列
 * 训练的完整实践", blog.gitcode.com, section "BigBird：从二次方注意力到线性稀疏
 * 注意力"): Q, K and V are cut into blocks of block_size tokens
 * (nb = L / block_size blocks).  The first and last blocks are global: query
 * blocks 0 and nb-1 attend every key block, and every query block attends
 * key blocks 0 and nb-1.  Every other query block i also attends its window
 * {i-1, i, i+1} and the r random blocks of row i of a per-head table.  The
 * attended set A(i) is a set (each key block once).  For key token u of an
 * attended block the score is
 *     s = scale * <q, k_u> + (key_mask[b][u] ? 0 : mask_value)
 * and the row softmax over the attended keys weights V.  Options (see
 * bb_attn_desc): seeded attention dropout on the attended probabilities,
 * and a query-side mask that zeroes the output rows of padding tokens.
 *
 * Conventions shared by every call:
 *  - All tensors are dense, row-major, contiguous.  Q, K, V, O, dO, dQ, dK
 *    and dV are [B][H][L][d] in the descriptor's dtype (fp32 or bf16; dQ,
 *    dK and dV in fp32 instead when grad_fp32 = 1); the blocked view
 *    [B][H][nb][block_size][d] of the pages is the same memory.
 *    lse and the workspace's fp32 arrays are fp32.
 *  - Pointers named *_host are host memory; every other pointer is device
 *    memory of the current CUDA device.  The caller owns every buffer; the
 *    library allocates nothing on the call path and keeps no state between
 *    calls.  Device pointers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Compute
 *    calls validate on the host, enqueue their kernels on `stream` and return
 *    without synchronising.  Launch errors are returned; faults detected by a
 *    kernel (a wait that ran out, a corrupt random table) are written to a
 *    status word at the start of the workspace, read by bb_attn_check_status.
 *  - Calls are re-entrant and thread-safe (no global mutable state; the one
 *    exception is bb_attn_fwd_noalloc's built-in scratch, see there); two
 *    calls may share a workspace only if they are ordered on the GPU.
 *  - Results are deterministic run to run: no floating-point atomics.
 */
#ifndef BB_ATTN_H_
#define BB_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BB_ABI_VERSION 5

#if defined(__GNUC__)
#define BB_API __attribute__((visibility("default")))
#else
#define BB_API
#endif

typedef enum {
  BB_OK = 0,
  BB_ERR_INVALID = -1,     /* a NULL or misaligned pointer, a bad size */
  BB_ERR_UNSUPPORTED = -2, /* valid but not built: d != 64, block_size not
                              in {32, 64, 128}, nb > 8192, r > 32 */
  BB_ERR_CUDA = -3,        /* a CUDA runtime call failed (launch, copy) */
  BB_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than required */
  BB_ERR_TIMEOUT = -5,     /* (status word) a bounded device wait ran out */
  BB_ERR_BAD_TABLE = -6    /* (status word) a random-table entry outside
                              [-1, nb) was found and ignored */
} bb_status;

typedef enum { BB_F32 = 0, BB_BF16 = 1 } bb_dtype;

/* Problem description.  d must be 64; block_size 32, 64 or 128 and a divisor
 * of L; r >= 0 random blocks per middle row; dtype a bb_dtype.
 * scale == 0 selects 1/sqrt(d) (key_dim = hidden / heads, as the pages'
 * layer sets it).  mask_value == 0 selects -10000, the pages' offset for
 * masked positions.  The scale multiplies <q, k> before the offset is added;
 * the offset is not scaled.
 *
 * dropout is the attention-dropout rate in [0, 1) ([gitcode page] sections
 * "BigBirdEncoder 的关键参数", attention_dropout_rate, and "梯度检查点的实现方式",
 * which asks for stateless seeded dropout so a recomputation draws the same
 * noise).  It acts on the attended softmax probabilities: kept ones are
 * multiplied by 1 / keep probability, dropped ones by 0; the lse output stays
 * that of the undropped softmax.  The rate is rounded to the nearest multiple
 * of 1/256 (thr = floor(256 rate + 1/2), keep probability (256 - thr) / 256);
 * a rate that rounds to 0 disables dropout, one that rounds to 1 is
 * BB_ERR_INVALID.  The keep decision of element (b, h, query token t, key
 * token u) is a pure function of dropout_seed and (b, h, t, u): Philox4x32-10
 * (Salmon, Moraes, Dror and Shaw, SC 2011) with counter words
 * (u >> 4, t, h, b) and key words (seed mod 2^32, seed >> 32) gives 16 bytes,
 * little-endian from its four output words in order, for key tokens
 * 16 (u >> 4) .. 16 (u >> 4) + 15; byte u & 15 keeps the element when it is
 * >= thr.  The backward must be called with the forward's dropout and
 * dropout_seed.
 *
 * mask_queries (0 or 1): with a key_mask, 1 also masks the query side, as
 * the pages' BigBirdMasks derives its from-side mask from the same input
 * mask ([gitcode page] "随机块掩码是如何生成的"): the output rows of padding
 * tokens are 0, so they pass no gradient (their dq rows are 0 and they add
 * nothing to dk, dv); their lse is still the row's normaliser.  The
 * backward must be called with the forward's mask_queries.  Ignored without
 * a key_mask.
 *
 * grad_fp32 (0 or 1; backward only): 1 writes dq, dk and dv as fp32 instead
 * of the dtype.  The kernels accumulate in fp32 either way; with bf16 the
 * stored gradient is that fp32 value rounded to nearest even, bit for bit.
 * Why it matters: the gradients of the two global key blocks sum over every
 * query row, so their magnitude grows with the square root of L (about 5
 * at L = 32768 and 10 at L = 131072 for unit-variance inputs), and above 4
 * bf16's own spacing (1/32, then 1/16 above 8) alone exceeds an absolute
 * error of 1e-2.  Use grad_fp32 = 1 where gradients must be within a fixed
 * absolute error of the exact result at such lengths.  Ignored for fp32
 * dtype (the gradients are fp32 already).
 *
 * dropout_bits (optional; NULL = off): a device buffer of
 * bb_attn_dropout_bits_size(desc) bytes, 16-byte aligned, owned by the
 * caller, that carries the dropout keep decisions from the forward to the
 * backward.  With a nonzero dropout rate, bb_attn_fwd writes there the
 * decisions it draws, and bb_attn_bwd reads them instead of drawing them
 * again (a Philox4x32-10 call per 16 elements in each of its two passes).
 * The decisions are the same either way, so the results are bit for bit
 * those of a call with dropout_bits = NULL; only the time differs.  The
 * buffer must hold what a forward with the same descriptor (dropout_seed
 * included), rand_idx and key_mask wrote, and must not be written between
 * that forward and the backward.  Entries of key tiles whose keys are all
 * masked may be left unwritten (their probabilities are 0, so their
 * decisions change nothing).  Used by the tensor-core kernels (bf16, the shapes listed for
 * them); the CUDA-core kernels neither write nor read it.  Ignored when the
 * rate rounds to 0.  Layout (a pure function of the descriptor and the
 * table): per (b, h), slots of block_size x block_size bits, one per
 * attended (query block i, key block u) pair, query row major with 32 keys
 * per uint32 word (bit j of word w of row q: key u * block_size + 32 w + j,
 * bit set = kept).  Slots of (b, h) start at word
 * (b * H + h) * S * block_size^2 / 32 with S = 2 nb + (nb - 2)(5 + r)
 * (S = 1 for nb = 1); query block 0 uses slot u, block nb - 1 slot nb + u,
 * and a middle block i slot 2 nb + (i - 1)(5 + r) + c(i, u), where c(i, u)
 * counts the members of {0, i - 1 if >= 2, i, i + 1 if <= nb - 2} and the
 * entries of table row i in [0, nb) that are below u. */
typedef struct {
  int B, H, L, d, block_size, r;
  int dtype;
  float scale;
  float mask_value;
  float dropout;
  uint64_t dropout_seed;
  int mask_queries;
  int grad_fp32;
  void* dropout_bits;
} bb_attn_desc;

/* Random block table ([gitcode page] section "随机块掩码是如何生成的": per
 * head, each middle row draws num_rand_blocks blocks among the middle blocks
 * outside its own window).  Writes int32 out_host[heads][num_blocks][r]:
 * rows 0 and num_blocks-1 are all -1; middle row i holds
 * r_eff = min(r, |cand(i)|) distinct ids from cand(i) = {j in [1, nb-2] :
 * |j - i| > 1}, sorted ascending, then -1 in the remaining slots.  The draw
 * is this library's own specification: a SplitMix64 stream (Steele, Lea and
 * Flood, OOPSLA 2014) seeded with seed ^ ((uint64)h << 32 | i) drives a
 * partial Fisher-Yates shuffle of cand(i) (slot k swaps with
 * k + u mod (|cand| - k)).  Deterministic and platform independent; host
 * only, no CUDA call.  Returns BB_ERR_INVALID for a NULL out_host (unless the
 * table is empty) or a negative size. */
BB_API int bb_rand_attn_build(uint64_t seed, int heads, int num_blocks, int r,
                       int32_t* out_host);

/* Random block table with the options of the pages' layer ([gitcode page]
 * section "随机块掩码是如何生成的": the table is fixed per head when the layer
 * is built, for its maximum length, with random blocks capped by
 * last_idx = 1024 tokens, and the first L / block_size - 2 middle rows are
 * used at run time; section "网络实现：从配置文件到编码器": the maximum
 * length is max_rand_mask_length = max_position_embeddings and the seed is
 * the layer index).
 *   max_blocks  rows are drawn as for a table of max_blocks blocks
 *               (max_rand_mask_length / block_size; >= num_blocks), and the
 *               first num_blocks rows are returned; 0 = num_blocks
 *   last_block  random candidates are restricted to ids < last_block
 *               (last_idx / block_size); 0 = no cap
 * Row i (0 < i < num_blocks - 1) draws, exactly as bb_rand_attn_build does
 * (same SplitMix64 stream and partial Fisher-Yates shuffle), r_eff =
 * min(r, |cand(i)|) ids from cand(i) = {j in [1, max_blocks - 2] :
 * |j - i| > 1, and j < last_block when last_block > 0}, then keeps those
 * <= num_blocks - 2, sorted
 * ascending, with -1 in the remaining slots.  Dropping an id past the
 * shorter table's middle blocks leaves the attended set unchanged (its last
 * block is global) or removes a block the sequence does not have.  With
 * max_blocks = 0 and last_block = 0 the result equals bb_rand_attn_build.
 * Returns BB_ERR_INVALID for a negative argument, max_blocks < num_blocks,
 * or a NULL out_host (unless the table is empty).  Host only. */
BB_API int bb_rand_attn_build_ex(uint64_t seed, int heads, int num_blocks, int r,
                                 int max_blocks, int last_block, int32_t* out_host);

/* Bytes of device workspace bb_attn_fwd (pass 0) or bb_attn_bwd (pass 1)
 * needs for `desc`; written to *bytes.  Host only. */
BB_API int bb_attn_workspace_size(const bb_attn_desc* desc, int pass, size_t* bytes);

/* Bytes of the optional dropout keep-bit buffer (bb_attn_desc.dropout_bits)
 * for `desc`: B * H * S * block_size^2 / 8 with S as given there (about 1
 * bit per attended probability); 0 when the dropout rate rounds to 0.
 * Written to *bytes.  Host only. */
BB_API int bb_attn_dropout_bits_size(const bb_attn_desc* desc, size_t* bytes);

/* Forward ([gitcode page] section "BigBird：从二次方注意力到线性稀疏注意力":
 * five segments first / second / middle / second_last / last, masked keys
 * offset by -10000, row softmax).
 *   q, k, v   [B][H][L][d] dtype, device
 *   key_mask  [B][L] uint8, nonzero = attend; NULL = attend every key
 *   rand_idx  [H][nb][r] int32, device (as bb_rand_attn_build writes it;
 *             entries of rows 0 and nb-1 are ignored, -1 is padding, other
 *             entries outside [0, nb) are ignored and flag BB_ERR_BAD_TABLE)
 *   out       [B][H][L][d] dtype, device (written)
 *   lse       [B][H][L] fp32, device (written): natural-log sum of exp of the
 *             row's attended scores, used by the backward
 *   workspace device, >= bb_attn_workspace_size(desc, 0) bytes */
BB_API int bb_attn_fwd(const bb_attn_desc* desc, const void* q, const void* k,
                const void* v, const uint8_t* key_mask,
                const int32_t* rand_idx, void* out, float* lse,
                void* workspace, size_t workspace_bytes, void* stream);

/* Backward: gradients of the forward's output for upstream gradient dout.
 * The pages train the layer by autodiff with recomputation (section
 * "梯度检查点的实现方式"); this computes the same gradient directly,
 * recomputing the probabilities from lse instead of storing them.
 *   q, k, v, out, lse, key_mask, rand_idx as produced / used by bb_attn_fwd
 *   dout      [B][H][L][d] dtype, device
 *   dq, dk, dv [B][H][L][d] dtype (fp32 when desc->grad_fp32 = 1), device
 *             (written)
 *   workspace device, >= bb_attn_workspace_size(desc, 1) bytes; holds the
 *             transposed block adjacency (query blocks per key block) and
 *             the per-row D = <dO, O>. */
BB_API int bb_attn_bwd(const bb_attn_desc* desc, const void* q, const void* k,
                const void* v, const void* out, const float* lse,
                const void* dout, const uint8_t* key_mask,
                const int32_t* rand_idx, void* dq, void* dk, void* dv,
                void* workspace, size_t workspace_bytes, void* stream);

/* The projections on either side of the attention in the pages' encoder
 * layer ([gitcode page] section "两条构建路径：EncoderScaffold 与
 * BigBirdEncoder": the layer is a transformer block around BigBirdAttention
 * with key_dim = hidden / heads), on tcgen05 tensor cores.  Head dim 64.
 * Weights follow the linear-layer convention W[out_features][in_features];
 * bias is fp32 [out_features] or NULL (no bias).  Accumulation is fp32; the
 * bf16 results are rounded to nearest even once.
 *
 * Fused Q/K/V projection: with D = H * 64,
 *   q[b][h][l][j] = b_qkv[h*64 + j]       + sum_c x[b][l][c] w_qkv[h*64 + j][c]
 *   k[b][h][l][j] = b_qkv[D + h*64 + j]   + sum_c x[b][l][c] w_qkv[D + h*64 + j][c]
 *   v[b][h][l][j] = b_qkv[2D + h*64 + j]  + sum_c x[b][l][c] w_qkv[2D + h*64 + j][c]
 *   x      [B][L][hidden] bf16, device
 *   w_qkv  [3 * H * 64][hidden] bf16, device;  b_qkv [3 * H * 64] fp32 or NULL
 *   q, k, v [B][H][L][64] bf16, device (written): the layout bb_attn_fwd reads
 * Requires L % 128 == 0, hidden % 64 == 0 and H % 4 == 0 (BigBird-base and
 * -large: hidden 768 / 1024, H 12 / 16), else BB_ERR_UNSUPPORTED.
 * workspace: device, >= 256 bytes, 16-byte aligned; holds the status word
 * (bb_attn_check_status).  Asynchronous on `stream`. */
BB_API int bb_qkv_proj(int B, int L, int hidden, int H, const void* x, const void* w_qkv,
                       const float* b_qkv, void* q, void* k, void* v, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Output projection of the attention output o [B][H][L][64] (as bb_attn_fwd
 * writes it):
 *   out[b][l][n] = b_o[n] + sum_{h, j} o[b][h][l][j] w_o[n][h*64 + j]
 *   w_o [hidden][H * 64] bf16, device;  b_o [hidden] fp32 or NULL
 *   out [B][L][hidden] bf16, device (written)
 * Requires L % 128 == 0 and hidden % 256 == 0, else BB_ERR_UNSUPPORTED.
 * workspace as for bb_qkv_proj. */
BB_API int bb_out_proj(int B, int L, int H, int hidden, const void* o, const void* w_o,
                       const float* b_o, void* out, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Number of kernel launches bb_attn_fwd (pass 0) or bb_attn_bwd (pass 1)
 * makes for `desc`, written to *launches.  Host only. */
BB_API int bb_attn_launch_count(const bb_attn_desc* desc, int pass,
                                int* launches);

/* Name of internal launch `index` (0-based, < bb_attn_launch_count) of
 * pass 0 (forward) or 1 (backward) for `desc`, as a static NUL-terminated
 * string in *name (e.g. "simt_fwd", "bwd_pre").  Host only. */
BB_API int bb_attn_launch_name(const bb_attn_desc* desc, int pass, int index,
                               const char** name);

/* Profiling variants of bb_attn_fwd / bb_attn_bwd: same arguments and
 * results, plus `events`, an array of num_events cudaEvent_t handles created
 * by the caller.  events[k] is recorded on `stream` just before internal
 * launch k and events[n] after the last one (n = bb_attn_launch_count);
 * entries beyond num_events are not recorded.  Lets a caller time each
 * kernel with CUDA events on the stream it runs on. */
BB_API int bb_attn_fwd_events(const bb_attn_desc* desc, const void* q,
                              const void* k, const void* v,
                              const uint8_t* key_mask,
                              const int32_t* rand_idx, void* out, float* lse,
                              void* workspace, size_t workspace_bytes,
                              void* stream, void* const* events,
                              int num_events);
BB_API int bb_attn_bwd_events(const bb_attn_desc* desc, const void* q,
                              const void* k, const void* v, const void* out,
                              const float* lse, const void* dout,
                              const uint8_t* key_mask,
                              const int32_t* rand_idx, void* dq, void* dk,
                              void* dv, void* workspace,
                              size_t workspace_bytes, void* stream,
                              void* const* events, int num_events);

/* Forward without a workspace, for callers that cannot allocate device
 * memory (a runtime that reserves its whole memory budget at start-up and
 * forbids later cudaMalloc, a plugin that must not bypass its host
 * framework's allocator, a C caller with no spare buffer to lend).  The
 * pages have no counterpart of this call: it is an interface convenience.
 * Same arguments, results and kernels as bb_attn_fwd, except that the
 * workspace is a 32 MiB scratch array built into the library, which every
 * device that loads the library keeps until the process exits.  The caller
 * still provides q, k, v, key_mask, rand_idx, out and lse.
 *  - Nothing is allocated: no cudaMalloc, cudaFree or allocating routine.
 *  - Every call looks up the scratch's device address (cudaGetSymbolAddress)
 *    in the CUDA context current on the calling thread, so the call serves
 *    whichever context is current (the runtime's primary context or a
 *    caller's own driver-API context on the device).  The first call in a
 *    context also loads the library's device code there; make that first
 *    call before any stream capture.
 *  - Returns BB_ERR_WORKSPACE, without launching anything, when the problem
 *    needs more than 32 MiB of workspace (bb_attn_workspace_size(desc, 0)).
 *  - Every call shares the one scratch array of the context, which keeps the
 *    last call's contents (the call clears its status word and writes
 *    everything else before reading it): calls that overlap on the GPU
 *    (other streams, other threads on the same device) race; order them on
 *    one stream.  The device status word of the last call (a bounded wait
 *    that ran out, a corrupt random table) is read with
 *    bb_attn_noalloc_status. */
BB_API int bb_attn_fwd_noalloc(const bb_attn_desc* desc, const void* q,
                               const void* k, const void* v,
                               const uint8_t* key_mask,
                               const int32_t* rand_idx, void* out, float* lse,
                               void* stream);

/* Status word left in the built-in scratch by the last bb_attn_fwd_noalloc
 * of the current context: waits for `stream`, then returns BB_OK,
 * BB_ERR_TIMEOUT or BB_ERR_BAD_TABLE (as bb_attn_check_status does for a
 * workspace), or BB_ERR_CUDA if the lookup or the copy failed.  Allocates
 * nothing.  Like the forward it reports on, it has no counterpart in the
 * pages. */
BB_API int bb_attn_noalloc_status(void* stream);

/* Waits for `stream`, then returns the status word the last call that used
 * `workspace` left there (BB_OK, BB_ERR_TIMEOUT or BB_ERR_BAD_TABLE), or
 * BB_ERR_CUDA if the copy itself failed. */
BB_API int bb_attn_check_status(const void* workspace, void* stream);

/* Static description of a status code (never NULL). */
BB_API const char* bb_status_str(int status);

/* Failure-detection self-test.  Launches one small kernel on `stream` that
 * waits on an mbarrier through the bounded wait every tensor-core kernel
 * uses (limit 2 s).  armed = 1: nothing completes the barrier, so the wait
 * runs out, writes BB_ERR_TIMEOUT into the status word at the start of
 * `workspace` (any buffer of >= 256 bytes, 16-byte aligned) and returns;
 * the kernel exits normally and the context stays usable.  armed = 0: the
 * barrier completes at once and the status word stays BB_OK.  Asynchronous:
 * read the result with bb_attn_check_status(workspace, stream).  Returns
 * BB_ERR_INVALID for a NULL, misaligned or short workspace or armed not 0/1,
 * BB_ERR_CUDA if the launch fails. */
BB_API int bb_debug_wait_probe(void* workspace, size_t ws_bytes, int armed,
                               void* stream);

/* BB_ABI_VERSION of the loaded library. */
BB_API int bb_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BB_ATTN_H_ */
