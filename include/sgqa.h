/* sgqa.h — C ABI of libsgqa.so: Sparse GQA (Step 5 Preview's full-context attention layer)
 * on NVIDIA B200 (sm_100a).
 *
 * What the layer computes. The pages give prose, not formulas; these are the readings used:
 *   mo.ai.kr, "Step 5 Preview agentic work design", section "model structure and training
 *   stability" — the full-context layers use Sparse GQA on top of Gated GQA; shared index keys
 *   are compressed per block of B = 8 tokens; every KV group selects its own relevant past
 *   context; the final setting is k = 4096 tokens, i.e. 512 blocks.
 *   ai.info, "StepFun illustrates the 92-block architecture of Step 5 Preview", section "Sparse
 *   GQA aims at a 1 million token context" — relevant past blocks are selected instead of the
 *   whole history; blocks of eight cut indexing and selection cost eightfold.
 *
 *   (1) compress  kbar[b,j,:] = (1/B) sum_{i<B} k_idx[b, jB+i, :]   for complete blocks j < T/B
 *   (2) select    per (b,t,g): c = floor(t/B) (own block); candidates j < c scored by
 *                 s_j = q_idx[b,t,g,:] . kbar[b,j,:]; keep the best m = min(k/B - 1, c) by
 *                 (s desc, j asc) plus the own block c; ascending, padded with -1 to k/B
 *   (3) attend    for each head h of group g = floor(h / (Hq/G)), over the selected tokens
 *                 U = {u <= t : floor(u/B) in S}: o = softmax_U(q[b,t,h] . k[b,u,g] / sqrt(d)) v
 *   (4) gate      out[b,t,h,:] = o * sigmoid(gate_logits[b,t,h,:])      (elementwise, bf16 RNE)
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous row-major with the
 *     batch index leading, and 16-byte aligned. bf16 tensors are passed as uint16_t bit patterns.
 *       q, gate_logits, out  [batch, T, Hq, d]      k, v   [batch, T, G, d]
 *       q_idx                [batch, T, G, d_idx]   k_idx  [batch, T, d_idx]
 *       kbar (fp32)          [batch, T/B, d_idx]    sel (int32) [batch, T, G, k/B]
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call only enqueues
 *     work on it: no host synchronisation, no allocation, no freeing.
 *   - `ws` is caller-owned device workspace of at least the size the matching *_workspace_size
 *     call returns (256-byte aligned; sgqa_compress_keys needs none). Its first 256 bytes hold a
 *     sticky device status word; zero it once with sgqa_reset_device_status before first use.
 *     Calls that share one ws must not overlap on the device.
 *   - The return value reports argument validation and launch errors only (sgqa_status).
 *     Errors found on the device (a selection naming a block outside [0, t/B], a bounded wait
 *     that ran out) are recorded in the status word; read it with sgqa_get_device_status after
 *     synchronising the stream. Once it records SGQA_ERR_TIMEOUT, the tensor-core kernels of every
 *     CTA and of later calls sharing that ws stop early and leave their outputs unwritten, until
 *     sgqa_reset_device_status.
 *   - Supported shapes (else SGQA_ERR_UNSUPPORTED): d in {64, 128}; d_idx in {32, 64};
 *     B in {1, 2, 4, 8, 16}; k % B == 0; Hq % G == 0 with 1 <= Hq/G <= 16; 128 % G == 0;
 *     1 <= T < 2^28; batch * T * Hq < 2^31. A trailing partial block is never a candidate.
 *   - Results are deterministic: the same inputs give the same bits, run after run.
 */
#ifndef SGQA_H
#define SGQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SGQA_OK = 0,
  SGQA_ERR_INVALID_ARG = 1,   /* null pointer, misaligned pointer, negative size, ... */
  SGQA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set above */
  SGQA_ERR_WORKSPACE = 3,     /* ws too small or misaligned */
  SGQA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  SGQA_ERR_TIMEOUT = 5,       /* device status: a bounded wait ran out */
  SGQA_ERR_DEVICE_CHECK = 6   /* device status: a device-side argument check failed */
} sgqa_status;

typedef struct {
  int batch; /* sequences */
  int T;     /* tokens per sequence (for decode: cache capacity) */
  int Hq;    /* query heads */
  int G;     /* KV groups; head h uses group h / (Hq / G) */
  int d;     /* head dim of q, k, v, gate, out */
  int d_idx; /* indexer dim of q_idx, k_idx, kbar */
  int B;     /* block size (tokens per compressed index key) */
  int k;     /* selection budget in tokens; k / B blocks including the own block */
} sgqa_dims;

/* Human-readable text of a status code (static storage). */
const char* sgqa_status_string(int status);

/* Library version and build target (static storage), e.g. "sgqa 0.1 sm_100a". */
const char* sgqa_version(void);

/* Bytes of workspace that sgqa_compress_keys, sgqa_select, sgqa_attend and sgqa_forward need
 * for these dims; 0 if the dims are invalid or unsupported. */
size_t sgqa_workspace_size(const sgqa_dims* dims);

/* Bytes of workspace sgqa_decode needs for n_new new tokens per sequence; 0 if invalid. */
size_t sgqa_decode_workspace_size(const sgqa_dims* dims, int n_new);

/* Zero the device status word at the start of ws (async on stream). */
int sgqa_reset_device_status(void* ws, size_t ws_bytes, void* stream);

/* Copy the device status word to *status (a blocking device-to-host copy; call after the
 * stream that ran the kernels has been synchronised). *status is SGQA_OK or an error code. */
int sgqa_get_device_status(const void* ws, size_t ws_bytes, int* status);

/* Step (1): block-mean compression of the shared index keys (see the header comment).
 * k_idx [batch, T, d_idx] bf16 -> kbar [batch, T/B, d_idx] fp32. The block's keys are summed
 * in fp64 in token order and rounded once, so kbar is the fp32 rounding (RNE) of the block
 * mean. This call uses no workspace: ws may be NULL and ws_bytes 0. With T < B there is no
 * complete block and kbar may be NULL. */
int sgqa_compress_keys(const sgqa_dims* dims, const uint16_t* k_idx, float* kbar, void* ws,
                       size_t ws_bytes, void* stream);

/* Step (2): per-(token, group) block selection.
 * q_idx [batch, T, G, d_idx] bf16, kbar [batch, T/B, d_idx] fp32 -> sel [batch, T, G, k/B]
 * int32: ascending block ids, own block last among the valid entries, -1 padding; exactly
 * min(k/B, floor(t/B) + 1) valid entries per row. Scores are accumulated in fp32; candidates
 * whose fp32 scores tie go to the lower block index. */
int sgqa_select(const sgqa_dims* dims, const uint16_t* q_idx, const float* kbar, int32_t* sel,
                void* ws, size_t ws_bytes, void* stream);

/* Steps (3)+(4): gated attention of every query row over a given selection.
 * q, gate [batch, T, Hq, d], k, v [batch, T, G, d] bf16; sel [batch, T, G, k/B] int32 in the
 * format sgqa_select writes: strictly ascending block ids <= t/B, then -1 padding (entries that
 * break this are flagged by a device check (SGQA_ERR_DEVICE_CHECK) and skipped)
 * -> out [batch, T, Hq, d] bf16. Rows are scheduled in tiles of rows with similar selections
 * (a deterministic function of sel); each tile gathers the union of its rows' blocks once. */
int sgqa_attend(const sgqa_dims* dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                const uint16_t* gate, const int32_t* sel, uint16_t* out, void* ws,
                size_t ws_bytes, void* stream);

/* The whole layer, steps (1)-(4), for all T rows of every sequence. If sel_out is not NULL it
 * receives the selection [batch, T, G, k/B]; otherwise the selection is kept in ws, in query
 * chunks (index selection chunked to bound memory, as the pages describe for training). */
int sgqa_forward(const sgqa_dims* dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 const uint16_t* q_idx, const uint16_t* k_idx, const uint16_t* gate,
                 uint16_t* out, int32_t* sel_out, void* ws, size_t ws_bytes, void* stream);

/* The layer for query rows [t_begin, t_end) of every sequence only: the unit of work when the
 * queries of one sequence are split over several GPUs (each GPU holds the whole sequence's k, v
 * and k_idx, gathered from all GPUs, and its own rows of q, gate and q_idx). The rows' results
 * are bit-identical to the same rows of sgqa_forward.
 *   q_rows, gate_rows, out_rows [batch, t_end - t_begin, Hq, d]; q_idx_rows [batch, t_end -
 *   t_begin, G, d_idx]; sel_out_rows (optional) [batch, t_end - t_begin, G, k/B];
 *   k, v [batch, T, G, d], k_idx [batch, T, d_idx] (whole sequences).
 * 0 <= t_begin <= t_end <= T (else SGQA_ERR_INVALID_ARG); ws as for sgqa_forward. */
int sgqa_forward_rows(const sgqa_dims* dims, int t_begin, int t_end, const uint16_t* q_rows,
                      const uint16_t* k, const uint16_t* v, const uint16_t* q_idx_rows,
                      const uint16_t* k_idx, const uint16_t* gate_rows, uint16_t* out_rows,
                      int32_t* sel_out_rows, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace sgqa_attend_backward needs; 0 if the dims are invalid or unsupported. */
size_t sgqa_backward_workspace_size(const sgqa_dims* dims);

/* Gradients of steps (3) and (4) through a given selection (the selection is a discrete choice
 * and carries no gradient; the pages train the 1M-context model with this layer: mo.ai.kr, "Step 5
 * Preview agentic work design", section "model structure and training stability"). With
 * z_u = q . k_u / sqrt(d), p = softmax over the selected tokens u <= t, o = sum p_u v_u,
 * s = sigmoid(gate) and dout the gradient of out = o * s:
 *   dgate = dout * o * s * (1 - s);  do = dout * s;  dz_u = p_u (do . v_u - do . o);
 *   dq = sum_u dz_u k_u / sqrt(d);  dk_u = sum over rows dz_u q / sqrt(d);  dv_u = sum over rows p_u do.
 * q, gate, dout [batch, T, Hq, d], k, v [batch, T, G, d] bf16; sel [batch, T, G, k/B] in
 * sgqa_select's format -> dq, dgate [batch, T, Hq, d] and dk, dv [batch, T, G, d], fp32 (every
 * element written). Deterministic: the same inputs give the same bits (no floating-point atomics).
 * Supported: d in {64, 128}, B in {4, 8, 16}, Hq/G <= 16 (else SGQA_ERR_UNSUPPORTED); ws of
 * sgqa_backward_workspace_size bytes, its first 256 bytes the status word as for the others. */
int sgqa_attend_backward(const sgqa_dims* dims, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const uint16_t* gate, const int32_t* sel,
                         const uint16_t* dout, float* dq, float* dk, float* dv, float* dgate,
                         void* ws, size_t ws_bytes, void* stream);

/* One decode step for dims.batch sequences sharing one cache length.
 * Caches (dims.T = capacity): k_cache, v_cache [batch, T, G, d], kidx_cache [batch, T, d_idx]
 * bf16, kbar_cache [batch, T/B, d_idx] fp32 holding the block means of every block complete in
 * the first cache_len tokens. New tokens: q_new, gate_new [batch, n_new, Hq, d], k_new, v_new
 * [batch, n_new, G, d], qidx_new [batch, n_new, G, d_idx], kidx_new [batch, n_new, d_idx].
 * The step writes the new k, v, k_idx rows at positions [cache_len, cache_len + n_new), adds
 * kbar for the blocks they complete, and writes out [batch, n_new, Hq, d] (and, if not NULL,
 * sel_out [batch, n_new, G, k/B]) for the last n_new rows of the concatenated sequence: the same
 * definition sgqa_forward computes for those rows, with the same selection rule, but not the same
 * arithmetic. Decode scores the candidates on its own kernels, so where two candidate scores
 * agree to within the rounding of the fp32 scores (a near-tie at the k/B-th place) decode and
 * forward may keep different blocks; elsewhere the selections are identical and the outputs agree
 * within the bf16 rounding. Requires cache_len + n_new <= T. Repeating a step at the same
 * cache_len rewrites the same rows and gives the same bits, so it is idempotent. */
int sgqa_decode(const sgqa_dims* dims, int cache_len, int n_new, uint16_t* k_cache,
                uint16_t* v_cache, uint16_t* kidx_cache, float* kbar_cache, const uint16_t* q_new,
                const uint16_t* k_new, const uint16_t* v_new, const uint16_t* qidx_new,
                const uint16_t* kidx_new, const uint16_t* gate_new, uint16_t* out,
                int32_t* sel_out, void* ws, size_t ws_bytes, void* stream);

/* FP8 storage of the KV cache (mo.ai.kr, "Step 5 Preview agentic work design", section
 * "long-horizon RL and run cost": the KV cache is trained for FP8 storage; the format is not given
 * there, this is the reading taken). Each (token, group) row of K or V is stored as d FP8 E4M3
 * codes plus one power-of-two scale s = 2^e per row, e the smallest integer with
 * max |x| <= 448 * s; a code is x / s rounded to the nearest E4M3 value (ties to even, 448 the
 * largest magnitude). code * s has at most 4 significant bits, so it is exact in bf16.
 * Quantizes rows [t0, t0 + n_t) of every sequence: src [batch, n_t, G, d] bf16 (the rows to
 * store) -> dst8 [batch, T, G, d] uint8 codes and dst_scale [batch, T, G] fp32 at positions
 * t0 .. t0 + n_t - 1 (dims->T = the caches' capacity). d must be 128 (else
 * SGQA_ERR_UNSUPPORTED); t0 + n_t <= T (else SGQA_ERR_INVALID_ARG). No workspace. */
int sgqa_quantize_kv_fp8(const sgqa_dims* dims, int t0, int n_t, const uint16_t* src, uint8_t* dst8,
                         float* dst_scale, void* stream);

/* sgqa_decode over FP8 K/V caches (format of sgqa_quantize_kv_fp8): k8_cache, v8_cache
 * [batch, T, G, d] codes with k_scale, v_scale [batch, T, G]; the step quantizes the n_new new K and
 * V rows into them (same rule), then computes the layer exactly as sgqa_decode would on caches
 * holding the dequantized values (selection: the index keys are not quantized, so it is
 * sgqa_decode's). Half the cache bytes of the bf16 step are gathered. Needs the tensor-core decode
 * attention: d = 128, B in {8, 16}, n_new * Hq/G <= 64, n_new * k/B <= 4096 (else
 * SGQA_ERR_UNSUPPORTED). Workspace: sgqa_decode_workspace_size. */
int sgqa_decode_fp8(const sgqa_dims* dims, int cache_len, int n_new, uint8_t* k8_cache, float* k_scale,
                    uint8_t* v8_cache, float* v_scale, uint16_t* kidx_cache, float* kbar_cache,
                    const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                    const uint16_t* qidx_new, const uint16_t* kidx_new, const uint16_t* gate_new,
                    uint16_t* out, int32_t* sel_out, void* ws, size_t ws_bytes, void* stream);

/* Gated SWA: the efficient attention layer that alternates 3:1 with the Sparse GQA layer
 * (mo.ai.kr, "Step 5 Preview agentic work design", section "model structure and training
 * stability"; ai.info, "StepFun illustrates the 92-block architecture of Step 5 Preview", section
 * "Why StepFun chose 92 transformer blocks"). The pages name the layer but give no window size;
 * it is the `window` argument here. For each (b, t) and head h of group g:
 *     U = {u : t - window < u <= t};  o = softmax_U(q[b,t,h] . k[b,u,g] / sqrt(d)) v;
 *     out[b,t,h,:] = o * sigmoid(gate_logits[b,t,h,:])                  (bf16 RNE)
 * i.e. the steps (3) and (4) above with a sliding window of keys in place of the selection.
 * q, k, v, gate, out as above; no index keys. The blocks the window overlaps are written as a
 * selection (ascending block ids, -1 padded) to sel_out [batch, T, G, k/B] if not NULL, else into
 * ws in chunks, and the tiled attention masks the tokens before the window.
 *   - dims->k is the selection row capacity in tokens: it must hold every block a window can
 *     overlap, so window >= B and dims->k >= window + B are required (else SGQA_ERR_INVALID_ARG).
 *   - Runs on the tcgen05 attention only: Hq/G in {4, 8, 16}, d in {64, 128}, B <= 16 (else
 *     SGQA_ERR_UNSUPPORTED).
 *   - ws as for sgqa_attend (sgqa_workspace_size(dims)). */
int sgqa_gated_swa(const sgqa_dims* dims, int window, const uint16_t* q, const uint16_t* k,
                   const uint16_t* v, const uint16_t* gate, uint16_t* out, int32_t* sel_out,
                   void* ws, size_t ws_bytes, void* stream);

/* Failure-detection test hook (host-side setting, not for production use). While cta >= 0, the
 * decode attention CTA with that grid index in later sgqa_decode / sgqa_decode_fp8 calls issues
 * no loads, so its tensor-core issuer's wait for the first tile is never satisfied: the wait
 * runs out after its bound (2 s), the kernel records SGQA_ERR_TIMEOUT in the status word and
 * returns with nothing in flight, and every other CTA and later kernel that polls that status
 * word stops early (until sgqa_reset_device_status). cta = -1 turns the hook off. Returns
 * SGQA_ERR_INVALID_ARG for cta < -1. Not thread-safe: set it while no other host thread calls. */
int sgqa_test_stall_decode_cta(int cta);

/* Size of the library-owned scratch array that sgqa_decode_noalloc uses (16 MiB). */
#define SGQA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* A decode step for callers that cannot allocate device memory. No counterpart on the pages:
 * this is a deployment variant of sgqa_decode, not a step of the method.
 * Same arguments, results and cache updates as sgqa_decode, but no ws: the step's scratch (status
 * word, indexer scores, selection, split-K partials) lives in one file-scope __device__ array of
 * SGQA_NOALLOC_SCRATCH_BYTES bytes that every GPU using the library holds until the process ends.
 * Nothing is allocated or freed: no cudaMalloc/cudaFree and no allocating library routine.
 *   - Returns SGQA_ERR_WORKSPACE if sgqa_decode_workspace_size(dims, n_new) exceeds
 *     SGQA_NOALLOC_SCRATCH_BYTES (e.g. 32 sequences at a 1M-token cache need more; use sgqa_decode),
 *     SGQA_ERR_INVALID_ARG / SGQA_ERR_UNSUPPORTED as sgqa_decode does.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *     that device current) and caches it; make that first call before any stream capture. The
 *     cached address belongs to the device's current context: resetting the device
 *     (cudaDeviceReset, or a reset of its primary context) while the library stays loaded
 *     invalidates it, and calling this entry point after such a reset is not supported.
 *   - Each call zeroes the status word (on `stream`) before its kernels; the device status is not
 *     readable through this entry point (use sgqa_decode with a workspace when it is needed).
 *   - All calls share the array and it keeps the last call's contents: calls that overlap on the
 *     GPU (other streams, other host threads) race; serialise them. */
int sgqa_decode_noalloc(const sgqa_dims* dims, int cache_len, int n_new, uint16_t* k_cache,
                        uint16_t* v_cache, uint16_t* kidx_cache, float* kbar_cache,
                        const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                        const uint16_t* qidx_new, const uint16_t* kidx_new,
                        const uint16_t* gate_new, uint16_t* out, int32_t* sel_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SGQA_H */
