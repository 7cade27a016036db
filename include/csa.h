/*
 * csa.h -- C ABI of the B200 (sm_100a) CSA/HCA compressed long-context
 * attention library (libcsa_b200.so).
 *
 * The layer it implements is described on these web pages (DeepSeek-V4
 * write-ups), cited below by short name:
 *   [cf-1]   cf-1.com/news/5231315, "企业官网建设流程全解析" (title as served):
 *            §3.1 "CSA 的工作方式", §3.2 "HCA 的工作方式", §3.3 "层间排布与滑窗补充",
 *            §3.4 "两个降开销的设计", §4.3 "确定性 Kernel", §4.4 "FP4 QAT 与 KV Cache 层级".
 *   [yfxerp] yfxerp.com/news/211352, "DeepSeek-V4 原理拆解：百万上下文之外，
 *            CSA/HCA/mHC/MegaMoE 强在哪", §3 config.toml skeleton
 *            ([attention.csa] / [attention.hca]).
 *
 * Conventions (all entry points):
 *  - Every tensor pointer is a DEVICE pointer into caller-owned memory; the
 *    library allocates nothing (except where an entry point says otherwise) and
 *    keeps no per-call state.  Tensors are dense row-major, last dim contiguous.
 *  - Every call only enqueues work on `stream` and returns a status; it never
 *    synchronises.  Arguments are validated on the host before any launch.
 *  - Floating tensors are CSA_F32 or CSA_BF16 (see each call); NVFP4 tensors are
 *    packed E2M1 bytes (element 2i in the low nibble, 2i+1 in the high nibble)
 *    plus one E4M3 scale byte per 16 elements plus one fp32 global scale g > 0.
 *  - Positions: q_pos0[b] (device, int32) is the absolute position of query row
 *    0 of sequence b (0 for a prefill, the cache length for decode).  Calls that
 *    take a row chunk [row0, row0 + T_chunk) place chunk row r at position
 *    p = q_pos0[b] + row0 + r; the others place query row r at q_pos0[b] + r.
 *  - Visibility: compressed entry s is visible at position p iff
 *    m*(s+1) - 1 <= p (only completed blocks are visible).
 *  - Raw window: raw token j is visible at p iff p - W < j <= p and j >= 0; it
 *    is stored at slot j % raw_cap of kv_raw [B, raw_cap, D] (raw_cap = T for a
 *    prefill, a ring of raw_cap >= W slots for decode).
 *  - Results are deterministic and batch-invariant: no atomics on outputs, no
 *    split reductions whose order depends on the launch ([cf-1] §4.3).
 *
 * Errors: CSA_ERR_INVALID_ARG (null pointer, bad size), CSA_ERR_UNSUPPORTED (a
 * shape outside the compiled set, e.g. a head dim the kernels do not handle),
 * CSA_ERR_ALIGNMENT (a pointer not 16-byte aligned), CSA_ERR_CUDA (the launch
 * failed; csa_last_cuda_error() returns the cudaError_t), CSA_ERR_TIMEOUT (a
 * bounded device wait gave up).  On any error nothing further is enqueued.
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa_stream_t; /* == cudaStream_t */

enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,
  CSA_ERR_UNSUPPORTED = 2,
  CSA_ERR_ALIGNMENT = 3,
  CSA_ERR_CUDA = 4,
  CSA_ERR_TIMEOUT = 5
};

enum { CSA_F32 = 0, CSA_BF16 = 1 };

/* Human-readable name of a status code (static string). */
const char* csa_status_string(int status);
/* cudaError_t of the most recent CSA_ERR_CUDA on the calling thread. */
int csa_last_cuda_error(void);
/* Library version as major*10000 + minor*100 + patch. */
int csa_version(void);
/* Device status words.  Kernels that wait on other warps of their CTA
 * (indexer_score, sparse_attn_fwd, hca_dense_attn_fwd) bound every wait in
 * wall time; a wait that gives up makes the kernel skip its remaining work and
 * return (it never traps) and stores CSA_ERR_TIMEOUT | (site << 8) into a
 * status word: the int32 `status` the call was given (device memory owned by
 * the caller, which sets it to 0 beforehand; the first failure is kept), or,
 * when the call passed NULL, the library's per-device word.
 * csa_device_status: synchronising read-and-clear of that per-device word
 * (CSA_OK or CSA_ERR_TIMEOUT | site << 8); CSA_ERR_CUDA if the copy fails. */
int csa_device_status(int* status_out);
/* Wall-time limit of every bounded device wait, in nanoseconds, for kernels
 * launched after the call (process-wide; 0 restores the default of 2 s). */
int csa_set_wait_timeout_ns(uint64_t ns);

/*
 * csa_compress -- gated overlapping m:1 KV compressor ([cf-1] §3.1: every 4
 * tokens become one entry; two KV streams mixed with softmax gate weights;
 * adjacent blocks share indices).
 *
 * For entry i with current block C = rows [m*i, m*i+m) and predecessor block
 * P = rows [m*(i-1), m*i), for each channel c:
 *   alpha = softmax over the 2m logits {z[t,c] : t in P u C}
 *   e[i,c] = sum_{t in C} alpha_t a[t,c] + sum_{t in P} alpha_t b[t,c]
 * Entry 0 has no predecessor and its softmax covers only its m logits.  A
 * trailing partial block emits nothing.
 *
 * Prefill mode (ring_pos == NULL): a, b, z are [B, T, D] (dtype in_dtype);
 * S = T/m - first_has_pred entries are written; with first_has_pred = 1 the
 * first m rows only serve as the predecessor block of the first entry.
 * Decode mode (ring_pos != NULL, device int32 [B]): a, b, z are rings
 * [B, 2m, D] holding raw token j at slot j % (2m); with p = ring_pos[b], if
 * (p+1) % m == 0 the entry i = (p+1)/m - 1 is written at entry index i of the
 * outputs (whose batch stride is out_bstride entries), else nothing is written
 * for that sequence.  An entry index i >= out_bstride (a full cache) is not
 * written.
 *
 * Outputs (either may be NULL, not both): out [B, out_bstride, D] in out_dtype;
 * NVFP4 out_fp4 [B, out_bstride, D/2] + out_sf [B, out_bstride, D/16] with
 * global scale gscale, quantised from the entry after rounding to out_dtype
 * (D % 16 == 0).  Prefill mode with out_bstride = 0 means out_bstride = S.
 * Requires D % 8 == 0, 1 <= m <= 16.
 */
int csa_compress(const void* a, const void* b, const void* z, int in_dtype,
                 int B, int T, int D, int m, int first_has_pred,
                 const int32_t* ring_pos, int out_bstride,
                 void* out, int out_dtype,
                 uint8_t* out_fp4, uint8_t* out_sf, float gscale,
                 csa_stream_t stream);

/*
 * hca_compress -- non-overlapping gated m:1 pooling ([cf-1] §3.2: 128 tokens
 * per entry, no overlap; [yfxerp] compress_ratio 128):
 *   e[i,c] = sum_{t in block i} softmax_{t in block i}(z[t,c]) * a[t,c]
 * a, z [B, T, D] in_dtype -> out [B, T/m, D] out_dtype.  D % 8 == 0, m >= 1.
 */
int hca_compress(const void* a, const void* z, int in_dtype,
                 int B, int T, int D, int m,
                 void* out, int out_dtype, csa_stream_t stream);

/*
 * nvfp4_quantize -- NVFP4 block quantisation of the indexer QK path ([cf-1]
 * §3.4: the indexer's QK runs in FP4; §4.4).  Along the last dim, blocks of 16:
 *   s_j = E4M3_rne_satfinite(amax_j / (6 g))        (fp32 division)
 *   q   = E2M1_rne_satfinite(x / (s_j * g))         (fp32 product, IEEE division)
 * q = 0 when s_j = 0.  x [rows, D] (CSA_F32 / CSA_BF16) -> packed [rows, D/2],
 * sf [rows, D/16].  D % 16 == 0, g > 0.  Bit-exact with the format definitions.
 */
int nvfp4_quantize(const void* x, int in_dtype, int64_t rows, int D, float gscale,
                   uint8_t* packed, uint8_t* sf, csa_stream_t stream);

/*
 * csa_decode_update -- one decode step's cache update in one launch (the
 * per-step work of [cf-1] §3.1 compression and §3.3 window for token p =
 * pos[b] of every sequence b), with the results of this call sequence:
 *   csa_ring_append of a, b, z, a_I, b_I, z_I into their 2m-slot carry rings,
 *   csa_compress (decode mode) of the KV entry into kv_c,
 *   csa_compress (decode mode, NVFP4 out) of the indexer key into k_fp4/k_sf,
 *   csa_ring_append of kv_raw into the W-slot window ring,
 *   nvfp4_quantize of q_I into q_fp4/q_sf (global scale gscale, also used
 *   for the keys).
 *   a, b, z, kv_raw [B, D]; a_I, b_I, z_I [B, DI]; q_I [B, HI, DI]   (this step)
 *   carry_* [B, 2m, D or DI], ring [B, W, D], kv_c [B, cap, D],
 *   k_fp4 [B, cap, DI/2], k_sf [B, cap, DI/16], q_fp4 [B, HI, DI/2], q_sf [B, HI, DI/16]
 * An entry whose index is >= cap is dropped.  Requires dtype CSA_BF16,
 * D and DI multiples of 16, DI <= 256 and (D/8 + 31)/32 + 1 + (HI DI/8 + 31)/32
 * <= 8 (else CSA_ERR_UNSUPPORTED; the separate calls serve other shapes);
 * 16-byte aligned rows, rings, q_I and kv_c.  pos is not advanced.
 */
int csa_decode_update(const void* a, const void* b, const void* z,
                      const void* a_I, const void* b_I, const void* z_I,
                      const void* kv_raw, const void* q_I, int dtype, int B,
                      int D, int DI, int HI, int m, int W, int cap,
                      void* carry_a, void* carry_b, void* carry_z,
                      void* carry_aI, void* carry_bI, void* carry_zI, void* ring,
                      void* kv_c, uint8_t* k_fp4, uint8_t* k_sf,
                      uint8_t* q_fp4, uint8_t* q_sf, float gscale,
                      const int32_t* pos, csa_stream_t stream);

/*
 * indexer_score -- lightning-indexer score over compressed entries ([cf-1]
 * §3.1 lightning indexer, §3.4 FP4 QK; [yfxerp] indexer_rank 64):
 *   score[b,r,s] = sum_h w[b,row0+r,h] * ReLU( qhat[b,row0+r,h,:] . khat[b,s,:] )
 * with qhat, khat the dequantised NVFP4 tensors (global scales q_g, k_g).
 * Runs on tcgen05 block-scaled FP4 MMA with fp32 accumulation.
 *   q_fp4 [B, T, HI, DI/2], q_sf [B, T, HI, DI/16], w fp32 [B, T, HI]
 *   k_fp4 [B, k_bstride, DI/2], k_sf [B, k_bstride, DI/16], entries s < S used
 *   score [B, T_chunk, score_ld] in score_dtype, rows r in [0, T_chunk) at
 *   positions q_pos0[b] + row0 + r.  Only visible (r, s) pairs are written.
 * Requires DI in {32, 64}, HI in {1, 2, 4, 8}, score_ld >= S; q_fp4 and k_fp4
 * 16-byte aligned, and k_sf 4-byte aligned when DI = 64 (else
 * CSA_ERR_ALIGNMENT).  status: optional device status word (see above).
 */
int indexer_score(const uint8_t* q_fp4, const uint8_t* q_sf, float q_gscale,
                  const uint8_t* k_fp4, const uint8_t* k_sf, float k_gscale,
                  const float* w, int B, int T, int row0, int T_chunk,
                  int S, int k_bstride, int HI, int DI, int m,
                  const int32_t* q_pos0, void* score, int score_dtype, int score_ld,
                  int32_t* status, csa_stream_t stream);

/*
 * topk_select -- per query row, the k largest visible scores ([cf-1] §3.1
 * top-k entries per query; [yfxerp] top_k_blocks).  Ties go to the smaller
 * entry index; +0 and -0 are equal.  Indices are written in ascending order;
 * when fewer than k entries are visible all of them are written, then -1.
 *   score [B, T_chunk, score_ld] (CSA_F32 / CSA_BF16), visible prefix of row r
 *   has n_r = min(S, (q_pos0[b] + row0 + r + 1) / m) entries
 *   idx int32 [B, T_chunk, k]
 * Radix select on order-preserving integer keys; bit-exact.  Scores must not
 * be NaN.
 * Workspace: topk_workspace_size() gives the bytes a shape can use (0 when it
 * needs none).  It is non-zero for few (B*T_chunk <= 512) long (S >= 16384)
 * rows, where BF16 rows are split across several CTAs that meet through the
 * workspace (4-byte aligned device memory owned by the caller; its contents
 * on entry do not matter, the call clears what it uses).  With workspace NULL
 * or smaller than that, the call falls back to one CTA per row (same result,
 * slower).  Calls that share a workspace must be ordered on one stream.
 */
int topk_select(const void* score, int score_dtype, int B, int T_chunk, int S,
                int score_ld, int k, int m, int row0, const int32_t* q_pos0,
                int32_t* idx, void* workspace, size_t ws_bytes,
                csa_stream_t stream);
size_t topk_workspace_size(int B, int T_chunk, int S, int k);

/*
 * indexer_topk -- indexer score and top-k selection in one kernel ([cf-1]
 * §3.1 the lightning indexer scores every visible compressed entry and each
 * query keeps its top-k; §4.4 the index score is BF16).  The result equals
 * topk_select applied to the BF16 scores indexer_score writes for the same
 * inputs, bit for bit (same arithmetic, rounding, keys, tie rule and output
 * order); the score matrix is never written.
 *   q_fp4, q_sf, w, k_fp4, k_sf, q_pos0, row0, T_chunk, S, m: as indexer_score
 *   idx int32 [B, T_chunk, k]: as topk_select
 * Requires DI = 64, HI in {4, 8} and S <= indexer_topk_max_entries(HI, DI)
 * (the visible scores of 8 query rows are held on chip), else
 * CSA_ERR_UNSUPPORTED: callers then use indexer_score + topk_select.  Same
 * alignment rules as indexer_score.  status: optional device status word
 * (see above).
 */
int indexer_topk(const uint8_t* q_fp4, const uint8_t* q_sf, float q_gscale,
                 const uint8_t* k_fp4, const uint8_t* k_sf, float k_gscale,
                 const float* w, int B, int T, int row0, int T_chunk,
                 int S, int k_bstride, int HI, int DI, int m,
                 const int32_t* q_pos0, int32_t* idx, int k,
                 int32_t* status, csa_stream_t stream);
/* Largest S indexer_topk accepts on the current device (0: HI/DI unsupported). */
int indexer_topk_max_entries(int HI, int DI);

/*
 * csa_validate_indices -- bounds check of an idx tensor before the attention
 * gathers with it (the layer drivers' check mode; [cf-1] §3.1: a query
 * attends to top-k entries among those it can see).  Row r of the chunk
 * (position p = q_pos0[b] + row0 + r) sees n = min(S, (p+1)/m) entries; a
 * valid row holds entries in [0, n), strictly ascending, then -1 padding.
 *   idx int32 [B, T_chunk, k]; status: caller device word
 * A violation writes CSA_ERR_INVALID_ARG | site << 8 to *status (the first
 * one is kept; site 1: entry outside [-1, n), 2: valid entries out of order,
 * 3: a valid entry after -1 padding).  The kernel only reads idx; it never
 * traps.
 */
int csa_validate_indices(const int32_t* idx, int B, int T_chunk, int k, int S,
                         int m, int row0, const int32_t* q_pos0,
                         int32_t* status, csa_stream_t stream);

/*
 * topk_select_noalloc -- topk_select for callers that cannot allocate device
 * memory (no workspace argument).  The pages have no counterpart to this call;
 * it exists only for allocator-free callers.  Same arguments, layouts, result
 * and statuses as topk_select with a workspace, except:
 *   - scratch: the multi-CTA path uses a fixed 1 MiB array inside the library
 *     (one per device per process) instead of caller memory; the call itself
 *     allocates nothing.  A shape whose multi-CTA histograms need more than
 *     1 MiB (topk_workspace_size() > 1048576) returns CSA_ERR_UNSUPPORTED and
 *     queues no work.  Shapes needing no scratch run the one-CTA-per-row path.
 *   - concurrency: calls that overlap in time on the same device (other
 *     streams, other host threads) share that scratch and race; order them.
 *   - set-up: the first call on a device (with that device current) looks up
 *     the scratch address; make it before any stream capture begins.  The
 *     address is kept for the life of the process, so after cudaDeviceReset
 *     this entry must not be called on that device again.
 */
int topk_select_noalloc(const void* score, int score_dtype, int B, int T_chunk,
                        int S, int score_ld, int k, int m, int row0,
                        const int32_t* q_pos0, int32_t* idx,
                        csa_stream_t stream);

/*
 * sparse_attn_fwd -- CSA attention ([cf-1] §3.1 sparse attention over the
 * selected compressed entries, §3.3 128-token raw window and attention sink).
 * For query row r (position p) and head h, over the key set
 *   J = { kv_c[b, s] : s in idx[b,r,:], s != -1 } u { raw j : p-W < j <= p, j >= 0 }
 * with key = value (MQA, one KV head):
 *   l_j = tau <q, key_j>,  M = max(sigma_h, max_j l_j)
 *   out = sum_j e^{l_j-M} key_j / (e^{sigma_h-M} + sum_j e^{l_j-M})
 *   lse = log sum_j e^{l_j}        (sink excluded; optional output)
 * sink == NULL means sigma = -inf.  W = 0 with sink == NULL gives the
 * compressed branch alone for swa_sink_merge.
 *   q, out [B, T, H, D] (rows row0 .. row0+T_chunk-1 are used), dtype
 *   kv_c [B, kv_bstride, D], idx int32 [B, T_chunk, k] (each row: its valid
 *   entries first, then -1 padding, as topk_select writes it), kv_raw [B, raw_cap, D]
 *   sink fp32 [H] or NULL, lse fp32 [B, T, H] or NULL
 * Requires D in {64, 128}.  bf16 runs on tcgen05 and needs D = 128, H in
 * {64, 128} and k <= 1024 (else CSA_ERR_UNSUPPORTED); fp32 runs on CUDA cores.
 * status: optional device status word (see above).
 */
int sparse_attn_fwd(const void* q, const void* kv_c, const int32_t* idx,
                    const void* kv_raw, const float* sink, float tau, int W,
                    int B, int T, int row0, int T_chunk, int H, int D,
                    int kv_bstride, int k, int raw_cap, const int32_t* q_pos0,
                    void* out, float* lse, int dtype, int32_t* status,
                    csa_stream_t stream);

/*
 * hca_dense_attn_fwd -- HCA attention ([cf-1] §3.2 dense attention over all
 * compressed entries, no selection; §3.3 window and sink): as sparse_attn_fwd
 * with the entry set = every visible entry s < S (m*(s+1) - 1 <= p).
 *   kv_c [B, kv_bstride, D]
 * bf16 needs D = 128 and H in {16, 32, 64, 128}; fp32 runs on CUDA cores.
 * status: optional device status word (see above).
 */
int hca_dense_attn_fwd(const void* q, const void* kv_c, const void* kv_raw,
                       const float* sink, float tau, int W,
                       int B, int T, int row0, int T_chunk, int H, int D,
                       int kv_bstride, int S, int m, int raw_cap,
                       const int32_t* q_pos0, void* out, float* lse,
                       int dtype, int32_t* status, csa_stream_t stream);

/*
 * swa_sink_merge -- the raw-window branch merged with a compressed-branch
 * result (o_c, lse_c) and the sink in one normalisation ([cf-1] §3.3):
 *   M = max(L_c, L_w, sigma_h)
 *   out = (e^{L_c-M} o_c + e^{L_w-M} o_w) / (e^{L_c-M} + e^{L_w-M} + e^{sigma_h-M})
 * where (o_w, L_w) is attention over the window alone.  Equals the fused
 * result of sparse_attn_fwd / hca_dense_attn_fwd.
 *   o_c, q, out [B, T, H, D] (dtype), lse_c fp32 [B, T, H], kv_raw [B, raw_cap, D]
 */
int swa_sink_merge(const void* o_c, const float* lse_c, const void* q,
                   const void* kv_raw, const float* sink, float tau, int W,
                   int B, int T, int row0, int T_chunk, int H, int D,
                   int raw_cap, const int32_t* q_pos0, void* out, int dtype,
                   csa_stream_t stream);

/*
 * grouped_out_proj -- the grouped output projection after the attention
 * ([cf-1] §3.4: with many query heads -- 128 -- the heads are split into
 * groups, each group's concatenated head outputs are projected to a smaller
 * dimension, and the concatenation of the groups is projected to the model
 * dimension, cutting the projection's parameters and FLOPs):
 *   y[:, j d_g : (j+1) d_g] = o[:, heads [j H/g, (j+1) H/g), :] . w1[j]^T
 *   out = y . w2^T
 *   o [M, H, D] bf16 (the attention output, M = B * T rows)
 *   w1 [groups, d_g, (H/groups) D] bf16, w2 [d_model, groups d_g] bf16
 *   y [M, groups d_g] bf16 (caller-owned intermediate), out [M, d_model] bf16
 * Two launches of one tcgen05 GEMM (fp32 accumulation in TMEM, bf16 stores);
 * y is rounded to bf16 between the products.  Requires (H/groups) D % 64 == 0,
 * d_g % 256 == 0 and d_model % 256 == 0 (else CSA_ERR_UNSUPPORTED), 16-byte
 * aligned tensors.  status: optional device status word (see above).
 */
int grouped_out_proj(const void* o, int M, int H, int D, int groups, int d_g,
                     const void* w1, const void* w2, int d_model, void* y,
                     void* out, int32_t* status, csa_stream_t stream);

/*
 * Decode-step helpers (state update of the KV cache tiers, [cf-1] §4.4):
 * csa_ring_append writes rows[b, :] (dtype, [B, D]) into ring[b, pos[b] % cap, :];
 * csa_pos_advance adds delta to each pos[b].  Both read positions on the device,
 * so a captured CUDA graph of a decode step stays valid from step to step.
 */
int csa_ring_append(const void* rows, int dtype, int B, int D, void* ring,
                    int cap, const int32_t* pos, csa_stream_t stream);
int csa_pos_advance(int32_t* pos, int B, int delta, csa_stream_t stream);

/*
 * csa_state_gather -- snapshots of a layer's decode-time state, the tier of
 * the KV cache that is not the compressed entries themselves ([cf-1] §4.4:
 * the sliding-window cache is checkpointed every 1024 tokens, so a request
 * that shares a prefix restores that state instead of recomputing it).  For
 * sequence b and snapshot c, with p = pos[b * npos + c] (the last token the
 * snapshot covers):
 *   window mode (m == 0): tokens j in (p - nrows, p]     (the raw window)
 *   carry mode  (m >= 1): tokens j in [m (floor((p+1)/m) - 1), p]  (the last
 *     complete block and the block in progress, which the next compressed
 *     entries mix)
 * are copied from src [B, src_cap, D] (token j at slot j % src_cap) into
 * dst [B, npos, dst_cap, D] at slot j % dst_cap; every other slot of dst, and
 * tokens j < 0, are written as zeros.  The same call restores a snapshot into
 * a decode ring: src = the snapshot (src_cap = dst_cap), npos = 1.
 * dtype CSA_F32 / CSA_BF16; D % 8 == 0; 16-byte aligned src and dst; dst_cap
 * >= nrows (window) or >= 2m (carry).  Device memory owned by the caller.
 */
int csa_state_gather(const void* src, int dtype, int B, int D, int src_cap,
                     const int32_t* pos, int npos, int m, int nrows,
                     void* dst, int dst_cap, csa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA_B200_H */
