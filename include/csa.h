/*
 * csa.h -- C ABI of libcsa_b200: the DeepSeek-V4 hybrid compressed attention layer on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (HF docs model_doc/deepseek_v4, section "Hybrid attention (2.3)"):
 *   1. a KV Compressor pools raw K=V rows into compressed entries by a per-channel
 *      softmax of gate logits over each window (CSA: ratio m=4, overlapping windows;
 *      HCA: ratio m'=128, non-overlapping)                         -> csa_compress
 *   2. the CSA Lightning Indexer scores every query against the causally visible
 *      entries and keeps the top-k                                  -> csa_index_topk
 *   3. single-KV-head shared K=V attention over the sliding window plus the selected
 *      entries (CSA) or every visible entry (HCA), with a per-head sink logit (eq. 27),
 *      interleaved-pair partial RoPE on the last rope_dim channels and the output's
 *      rope slice rotated back by -position (eq. 26)        -> csa_attend / hca_attend
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller; all tensors are dense
 *    row-major (innermost dimension last).  The library never allocates, frees or
 *    synchronises: every call only enqueues work on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) and returns.
 *  - `dtype` gives the element type of every floating tensor argument except `sink`
 *    (always fp32) and `scores_opt` (always fp32).  Arithmetic is fp32 throughout;
 *    bf16 tensors are rounded to nearest-even on store.
 *  - Positions are absolute token positions.  Query row i is at q_pos0 + i; raw K=V
 *    row r is at kv_pos0 + r; compressed entry j covers tokens ending at (j+1)*ratio-1,
 *    is visible to the query at t iff (j+1)*ratio - 1 <= t, and is rotated at position
 *    j*ratio.  All sequences of a batch share the positions.
 *  - Errors: arguments are checked on the host before anything is enqueued; a bad
 *    argument returns CSA_ERR_INVALID_ARG (or CSA_ERR_UNSUPPORTED for a valid shape
 *    this build does not handle, CSA_ERR_WORKSPACE for a short workspace) and
 *    csa_last_error() describes it.  A failed launch returns CSA_ERR_CUDA.  Kernels
 *    never trap.  Tensor pointers must be 16-byte aligned (idx and sink: 4-byte).
 *  - Shape limits of this build: D % 8 == 0 and 8 <= D <= 1024; rope_dim even and
 *    <= min(D, 256); 1 <= topk <= 2048; d_I % 8 == 0 and d_I <= 256; H, H_I >= 1.
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype_t;

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = -1,
    CSA_ERR_UNSUPPORTED = -2,
    CSA_ERR_CUDA = -3,
    CSA_ERR_WORKSPACE = -4
} csa_status_t;

/*
 * csa_compress -- KV Compressor (HF docs model_doc/deepseek_v4 section 2.3.1: CSA pools
 * with ratio m=4 over overlapping windows; section 2.3.2: HCA pools with m'=128 over
 * non-overlapping windows; HF PR #45616, compressor note: the module returns a tensor,
 * empty before the first window closes).
 *
 *   pool[b,j,d] = sum_{s in Win_j} softmax_{s in Win_j}(gate[b,s,d]) * kv[b,s,d]
 *   Win_j = [max(0,(j-1)*ratio), (j+1)*ratio) if overlap, else [j*ratio, (j+1)*ratio)
 *   for j in [0, P), P = floor(S / ratio); a trailing partial window is not emitted.
 *
 *   kv, gate : [B, S, D]   raw K=V rows (un-rotated) and gate logits, positions 0..S-1
 *   pool     : [B, P, D]   output, un-rotated; nothing is written when P == 0
 *   ratio >= 1; overlap in {0, 1}.
 */
csa_status_t csa_compress(const void *kv, const void *gate, void *pool, int64_t B, int64_t S,
                          int32_t D, int32_t ratio, int32_t overlap, csa_dtype_t dtype,
                          void *stream);

/*
 * csa_compress_append -- decode-time compressor cache update (HF PR #45616, note on
 * compressor and indexer state: each layer keeps, per compressor, a buffer of raw kv and
 * gate rows and the pooled cache, and one call accumulates the new rows and updates the
 * pool once; HF docs model_doc/deepseek_v4 section "Cache layers": buffer, pool, counter,
 * plus the overlap state for CSA).  The same call serves the main compressor (D = head_dim)
 * and the indexer's key compressor (D = d_I), each with its own state.
 *
 * Appends the raw rows of positions pos0 .. pos0+n_new-1 of every sequence and writes each
 * pool entry whose window closes among them -- entries j with pos0 <= (j+1)*ratio - 1 <
 * pos0 + n_new -- with the value csa_compress gives over the whole sequence.  Other pool
 * entries are not touched.
 *
 *   kv_new, gate_new : rows of sequence b at kv_new + b*kv_stride*D (gate: gate_stride),
 *                      n_new consecutive rows of D elements each; strides are in rows and
 *                      must be >= n_new when B > 1 (a view of a larger cache is fine)
 *   state  : [B, 2, L, D], L = (1+overlap)*ratio, csa_compress_state_bytes() bytes, owned
 *            by the caller: [b,0,p mod L,:] is the kv row of position p, [b,1,p mod L,:]
 *            its gate.  The call reads the rows of positions [max(0, pos0-L+1), pos0),
 *            which earlier calls must have stored (every call stores its newest
 *            min(n_new, L) rows); its initial contents are never read at pos0 == 0.
 *   pool   : [B, pool_cap, D], or NULL to store rows into the state only (e.g. to seed it
 *            from the tail of a prefill that csa_compress pooled); requires
 *            pool_cap >= floor((pos0+n_new)/ratio).
 *   pos0   : tokens appended so far (the compressor's counter), the same for every
 *            sequence.
 * A call that closes more than ~500K entries returns CSA_ERR_UNSUPPORTED (csa_compress is
 * the prefill path).
 */
csa_status_t csa_compress_append(const void *kv_new, const void *gate_new, int64_t kv_stride,
                                 int64_t gate_stride, void *state, void *pool, int64_t pool_cap,
                                 int64_t B, int64_t n_new, int64_t pos0, int32_t D,
                                 int32_t ratio, int32_t overlap, csa_dtype_t dtype, void *stream);

/* Bytes of the state csa_compress_append keeps for these sizes (0 for bad arguments). */
size_t csa_compress_state_bytes(int64_t B, int32_t D, int32_t ratio, int32_t overlap,
                                csa_dtype_t dtype);

/*
 * csa_index_topk -- CSA Lightning Indexer and top-k (HF docs model_doc/deepseek_v4
 * section 2.3.1, eq. 13-17 named there; section "Attention mask layout": queries before
 * the first closed window get only the -1 marker).
 *
 *   score[t,j] = sum_{h < H_I} w[b,i,h] * max(0, <q_I[b,i,h,:], k_I[b,j,:]>)
 *   for the visible entries j < n_vis(t) = min(P, floor((t+1)/ratio)), t = q_pos0 + i.
 *   idx[b,i,:] = the min(topk, n_vis) best entries (ranked by score descending, equal
 *   scores by lower j first), listed in ascending entry order, then -1 padding.
 *
 *   q_I : [B, S_q, H_I, d_I]   w : [B, S_q, H_I]   k_I : [B, P, d_I]
 *   idx : [B, S_q, topk] int32 output
 *   scores_opt : NULL, or [B, S_q, topk] fp32 output holding each kept entry's score
 *                (NaN in the -1 slots)
 *   workspace  : device scratch of at least csa_index_topk_workspace_bytes(...) bytes
 *                (may be NULL when that is 0); contents are not preserved.
 */
csa_status_t csa_index_topk(const void *q_I, const void *w, const void *k_I, int64_t B,
                            int64_t S_q, int64_t q_pos0, int64_t P, int32_t H_I, int32_t d_I,
                            int32_t ratio, int32_t topk, int32_t *idx, float *scores_opt,
                            void *workspace, size_t workspace_bytes, csa_dtype_t dtype,
                            void *stream);

/*
 * csa_rope_rows -- interleaved-pair partial RoPE over rows, for the Lightning Indexer's
 * own rotary embedding (TransformerLens deepseek_v4 bridge: the indexer's submodules
 * include a rotary embedding; HF PR #45616, note on the RoPE application: interleaved
 * channel pairs are rotated; HF docs model_doc/deepseek_v4 section 2.3.3).  With it the indexer scores rotated queries
 * against rotated pooled keys, so a score depends on t - j*ratio:
 *
 *   out[r] = Rot(x[r], pos0 + ((r / group) mod period) * step),  r in [0, rows)
 *   Rot: pairs (D-R+2i, D-R+2i+1) turned by pos * rope_base^(-2i/R), R = rope_dim; the
 *        first D-R channels are copied unchanged.
 *
 * Rows are taken in memory order.  Indexer queries q_I [B,S_q,H_I,d_I]: rows =
 * B*S_q*H_I, group = H_I, period = S_q, step = 1, pos0 = q_pos0.  Pooled index keys
 * k_I [B,P,d_I]: rows = B*P, group = 1, period = P, step = ratio, pos0 = 0 (entry j at
 * j*ratio, as the attention rotates entries).  Call it on both before csa_index_topk.
 *   x, out : [rows, D] device buffers; out may be x (in place) but must not otherwise
 *            overlap it.  D % 8 == 0, rope_dim even and <= min(D, 256); every position
 *            must stay within +-2^31.
 */
csa_status_t csa_rope_rows(const void *x, void *out, int64_t rows, int32_t D, int32_t rope_dim,
                           double rope_base, int64_t pos0, int64_t group, int64_t period,
                           int64_t step, csa_dtype_t dtype, void *stream);

/* Scratch bytes csa_index_topk needs for these sizes (0 when the call needs none).  When
 * every row has at most 16384 visible entries, the indexer writes every visible entry's
 * 32-bit score key to the workspace (one row of round_up(P, 4) keys per query) and a
 * selection kernel picks the top-k: decode-sized calls, and prefill calls whose key rows
 * take at most 2 GiB.  Otherwise a decode-sized call split over entry ranges passes each
 * range's candidates to a merge kernel, and a prefill call keeps its candidates in shared
 * memory (no workspace). */
size_t csa_index_topk_workspace_bytes(int64_t B, int64_t S_q, int64_t q_pos0, int64_t P,
                                      int32_t H_I, int32_t d_I, int32_t ratio, int32_t topk,
                                      csa_dtype_t dtype);

/*
 * csa_attend -- CSA attention: shared K=V single-head MQA over the sliding window plus
 * the selected entries, with sink, partial RoPE and output de-rotation (HF docs
 * model_doc/deepseek_v4 section 2.3: one K=V head shared by all query heads; section
 * 2.3.3 and eq. 26: partial RoPE, and the output's rope slice turned back by the query's
 * position; eq. 27: one learned sink logit per head; the sliding window as an extra
 * branch of keys; HF PR #45616: the eager attention is the GPT-OSS one, with the output
 * rope slice un-rotated).
 *
 * For query row i at t = q_pos0 + i, head h:
 *   keys K_t = { raw rows r : t - window < kv_pos0 + r <= t, 0 <= r < S_kv }
 *            + { pool entries idx[b,i,c] : idx[b,i,c] in [0, n_vis(t)) }  (other values,
 *              including -1, are skipped; an entry listed twice counts twice, and so
 *              does an entry whose tokens are also in the window)
 *   Rot(x, p): pairs (D-R+2i, D-R+2i+1) of x turned by p * rope_base^(-2i/R), R=rope_dim
 *   l_x = scale * <Rot(q[b,i,h], t), Rot(key_x, pos_x)>, pos_x = kv_pos0 + r or j*ratio
 *   M = max(max_x l_x, sink[h]),  Z = exp(sink[h] - M) + sum_x exp(l_x - M)
 *   out[b,i,h,:] = sum_x exp(l_x - M) / Z * Rot(key_x, pos_x), then its last R channels
 *                  are rotated by -t.
 *
 *   q   : [B, S_q, H, D]        kv : [B, S_kv, D] (un-rotated)   pool : [B, P, D]
 *   idx : [B, S_q, topk] int32  sink : [H] fp32 (may hold -INFINITY)
 *   out : [B, S_q, H, D] output
 *   workspace : device scratch of at least csa_attend_workspace_bytes(...) bytes.
 *   Requires q_pos0 >= 0 when S_q > 0 and window >= 1.
 * The tensor-core path (bf16, H = 64, D = 512, rope_dim <= 64) reads kv and pool in place
 * for decode-sized calls (S_q * 64 < S_kv + P); these take it when both pointers are
 * 16-byte aligned, and the general path otherwise.
 */
csa_status_t csa_attend(const void *q, const void *kv, int64_t S_kv, int64_t kv_pos0,
                        const void *pool, int64_t P, const int32_t *idx, int32_t topk,
                        const float *sink, void *out, int64_t B, int64_t S_q, int64_t q_pos0,
                        int32_t H, int32_t D, int32_t rope_dim, double rope_base,
                        int32_t window, int32_t ratio, float scale, void *workspace,
                        size_t workspace_bytes, csa_dtype_t dtype, void *stream);

/*
 * hca_attend -- HCA attention (HF docs model_doc/deepseek_v4 section 2.3.2: no indexer,
 * the query attends to every compressed entry; section "Attention mask layout": entry w
 * is visible to the query at t iff w < (t+1)//m).  Same as csa_attend with K_t's entry
 * part replaced by every visible entry j < n_vis(t).  P == 0 gives the sliding-window-only
 * layer.
 */
csa_status_t hca_attend(const void *q, const void *kv, int64_t S_kv, int64_t kv_pos0,
                        const void *pool, int64_t P, const float *sink, void *out, int64_t B,
                        int64_t S_q, int64_t q_pos0, int32_t H, int32_t D, int32_t rope_dim,
                        double rope_base, int32_t window, int32_t ratio, float scale,
                        void *workspace, size_t workspace_bytes, csa_dtype_t dtype,
                        void *stream);

/*
 * csa_attend_noalloc -- csa_attend for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for users of this library.
 *
 * Some callers cannot call cudaMalloc or pass a scratch buffer: a custom operator
 * inside a host framework that hands the operator only its input and output buffers
 * and owns every other byte of device memory through its own allocator (a raw
 * cudaMalloc would bypass its accounting and can fail under its memory budget), or a
 * latency-critical serving loop that must not allocate per call because cudaMalloc can
 * synchronise the device.  This entry point takes the same arguments as csa_attend
 * minus the workspace and allocates nothing: its scratch (the rotated window rows and
 * compressed entries and the rotated query chunks of the call) lives in one fixed device
 * array of 16 MiB compiled
 * into the library, created on each GPU that loads the library and held until the
 * process exits.  The caller still provides q, kv, pool, idx, sink and out.
 *
 *  - Handles the bf16, H = 64, D = 512 prefill shape (S_q * 64 >= S_kv + P) whose
 *    scratch fits the array: B * (S_kv + P) rotated key rows of 1 KB plus B * S_q * 64
 *    rotated query chunks of 128 B (each part rounded up to 256 B) within 16 MiB, e.g.
 *    B = 1, S_q = S_kv = 1024, P = 256 (9.3 MiB); anything else returns
 *    CSA_ERR_UNSUPPORTED with a message naming the limit.
 *  - The first call on a device looks up the array's device address (set-up, once per
 *    device, with that device current); make that first call before any stream capture.
 *  - Every call on a device shares the one array, and it keeps the last call's contents
 *    (every row a call reads is written by that call first).  Calls whose work overlaps
 *    on the GPU (different streams, or different host threads) race on it: serialise
 *    them, e.g. on one stream.
 */
csa_status_t csa_attend_noalloc(const void *q, const void *kv, int64_t S_kv, int64_t kv_pos0,
                                const void *pool, int64_t P, const int32_t *idx, int32_t topk,
                                const float *sink, void *out, int64_t B, int64_t S_q,
                                int64_t q_pos0, int32_t H, int32_t D, int32_t rope_dim,
                                double rope_base, int32_t window, int32_t ratio, float scale,
                                csa_dtype_t dtype, void *stream);

/*
 * csa_out_proj -- grouped low-rank output projection after the attention (HF docs
 * model_doc/deepseek_v4, section 2.3 "Grouped Output Projection": o_groups head groups,
 * o_lora_rank features per group by DeepseekV4GroupedLinear (o_a_proj), then o_b_proj to
 * hidden_size; HF PR #45616 on DeepseekV4GroupedLinear as a per-group batched matmul).
 *
 *   z[m, g*r + i] = sum_c o[m, g*(H/G)*D + c] * w_a[g, i, c]      (group g: heads
 *                   [g*H/G, (g+1)*H/G), flattened head-major, c < (H/G)*D)
 *   y[m, n]       = sum_k z[m, k] * w_b[n, k]
 *
 *   o   : [M, H, D]  the de-rotated attention output (M = B*S rows)
 *   w_a : [G, r, (H/G)*D]   w_b : [hidden, G*r]   y : [M, hidden] output
 *   workspace : at least csa_out_proj_workspace_bytes(M, G, r) bytes; it receives z in
 *               bf16 [M, G*r] (rounded there, fp32 accumulation in both products).
 * bf16 only.  Shape limits: (H/G)*D and G*r multiples of 64; r and hidden multiples of
 * 256 (CSA_ERR_UNSUPPORTED otherwise).
 */
csa_status_t csa_out_proj(const void *o, const void *w_a, const void *w_b, void *y, int64_t M,
                          int32_t H, int32_t D, int32_t G, int32_t r, int32_t hidden,
                          void *workspace, size_t workspace_bytes, csa_dtype_t dtype,
                          void *stream);

/* Scratch bytes csa_out_proj needs (the bf16 group features z). */
size_t csa_out_proj_workspace_bytes(int64_t M, int32_t G, int32_t r);

/*
 * csa_kv_gate_proj -- the compressor's input projections (TransformerLens deepseek_v4
 * bridge: the compressor carries kv_proj, gate_proj and kv_norm): per token row m,
 *
 *   kv[m, :]   = RMSNorm(x[m, :] . w_kv^T) * kv_norm_w,  RMSNorm(v) = v / sqrt(mean(v^2) + eps)
 *   gate[m, :] = x[m, :] . w_gate^T
 *
 * i.e. the raw K=V rows and gate logits csa_compress pools (the synthetic workloads feed
 * csa_compress RMS-normalised rows, which is what this produces with kv_norm_w = 1).
 *
 *   x : [M, hidden]   w_kv, w_gate : [D, hidden]   kv_norm_w : [D]
 *   kv, gate : [M, D] outputs
 * bf16 only (fp32 accumulation and normalisation).  Shape limits: hidden % 64 == 0,
 * D in {256, 512} (CSA_ERR_UNSUPPORTED otherwise).
 */
csa_status_t csa_kv_gate_proj(const void *x, const void *w_kv, const void *w_gate,
                              const void *kv_norm_w, float eps, void *kv, void *gate, int64_t M,
                              int32_t hidden, int32_t D, csa_dtype_t dtype, void *stream);

/* Scratch bytes csa_attend (mode 0) or hca_attend (mode 1) needs for these sizes. */
size_t csa_attend_workspace_bytes(int32_t mode, int64_t B, int64_t S_q, int64_t S_kv,
                                  int64_t P, int32_t H, int32_t D, int32_t topk,
                                  csa_dtype_t dtype);

/* Message for the last error returned on the calling host thread ("" if none). */
const char *csa_last_error(void);

/* Nonzero if a kernel of this library gave up on a bounded wait (and skipped the rest
 * of its work) since the last call; bit 0: attention, bit 1: indexer, bit 2: projections.  Synchronises the device and
 * clears the flags.  For tests and diagnostics. */
uint32_t csa_device_status(void);

/*
 * csa_debug_withhold_attention_loads -- test hook for the bounded-wait error path of the
 * tensor-core attention; not part of the layer (the pages have no counterpart).
 * on != 0: from the next launch on, the attention kernel's loader publishes nothing, so
 * every wait on it gives up after a short bound (well under a millisecond); the kernel
 * then skips its work (out is left unwritten or holds partial values), frees its tensor
 * memory, returns and sets bit 0 of csa_device_status().  Nothing faults or hangs and the
 * context stays usable.  on == 0 restores normal operation.  A process-wide host flag,
 * passed to every attention launch enqueued after the call (a CUDA graph captured
 * earlier keeps the value it was captured with).  Always returns CSA_OK.
 */
csa_status_t csa_debug_withhold_attention_loads(int32_t on);

/* Number of kernels this library has enqueued in this process (all devices, all
 * threads); for accounting launches in a timed region. */
uint64_t csa_launch_count(void);

/* Library version string. */
const char *csa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_B200_H */
