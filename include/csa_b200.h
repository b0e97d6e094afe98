/*
 * csa_b200.h -- C ABI of the B200 (sm_100a) Compressed Sparse Attention
 * (CSA) / Heavily Compressed Attention (HCA) library, libcsa_b200.so.
 *
 * The method, from the pages this library follows:
 *   "DS-V4 分析&学习" §1.2: CSA compresses every m tokens into one KV entry,
 *     a Lightning Indexer scores the entries, each query keeps its top-k and
 *     attends to those k compressed entries plus a sliding window of raw KV;
 *     §1.3: an entry sees 2m adjacent positions (neighbouring blocks
 *     overlap); §1.4: HCA compresses 128:1 and attends densely; §4: the
 *     indexer QK path runs in low precision.
 *   "百万上下文从「奢侈品」变「日用品」…" §3.2: compression is a mean pool over
 *     the block followed by a projection, floor(n/m) entries, the indexer is
 *     a dot product followed by a per-query top-k; §5.2: the window of query
 *     i is [max(0, i-W+1), i] and scores are scaled by 1/sqrt(head_dim).
 *   "DeepSeek V4 CSA + CP 迁移到 HP：困难点深度分析" §3.2: ratio 4 compresses
 *     with overlap, ratio 128 without; §7.2: the indexer has a compressor of
 *     its own, sharing the main compressor's entry index space.
 *
 * Conventions shared by every entry point
 *   - Tensor arguments are DEVICE pointers to caller-owned memory; the
 *     library never allocates, frees or keeps them.  Layouts are batch-first,
 *     contiguous, last dimension innermost.  Data tensors (activations,
 *     weights, caches, outputs) must start on a 16-byte boundary;
 *     per-element arrays (scales, gate weights, APE, compressor state,
 *     indices, positions, counts, LSE, block tables) on a 4-byte one (else
 *     CSA_ERR_MISALIGNED).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream).  Arguments are validated on the host first; on any
 *     error nothing is launched.  A launch failure returns CSA_ERR_CUDA.
 *     No call aborts, exits or throws; the text of the last error of the
 *     calling thread is returned by csa_last_error_detail().
 *   - Device index arrays that the host cannot read (n_entries, q_pos,
 *     raw_pos0, raw_len, idx) are clamped by the kernels to the buffers'
 *     extents, so a bad value never reads out of bounds.
 *   - Results are deterministic: the same inputs give bit-identical outputs.
 *   - Positions: a query row carries the absolute position t of its token
 *     (q_pos; NULL means t = the row's index q, i.e. a prefill from 0).
 *     Compressed entry i covers positions up to m(i+1)-1 and is visible to t
 *     iff i < min(floor((t+1)/m), n_entries[b]).  Raw row j of batch element
 *     b holds position raw_pos0[b]+j for 0 <= j < raw_len[b]; positions < 0
 *     are never attended (a partly filled sliding-window cache).
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad combination */
    CSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (dtype, head count, size) */
    CSA_ERR_MISALIGNED = 3,   /* a pointer breaks the alignment rule below */
    CSA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    CSA_ERR_TIMEOUT = 5       /* reserved: a bounded device-side wait expired */
} csa_status_t;

typedef enum {
    CSA_DT_F32 = 0,   /* IEEE binary32 */
    CSA_DT_BF16 = 1,  /* bfloat16 */
    CSA_DT_E4M3 = 2,  /* OCP FP8 E4M3 with one fp32 scale per row */
    CSA_DT_E4M3_HADAMARD = 3  /* as CSA_DT_E4M3, of rows rotated first by the normalised
                                 Walsh-Hadamard matrix (indexer keys; see csa_compress) */
} csa_dtype_t;

/* Static text of a status code ("CSA_OK", ...). */
const char* csa_status_string(int status);

/* Thread-local detail of the last non-OK return on the calling thread ("" if none). */
const char* csa_last_error_detail(void);

/* ABI version: 100 * major + minor. */
int csa_version(void);

/* Number of kernels this library has launched in the process so far
 * (diagnostics: lets a caller count the device work behind its calls). */
unsigned long long csa_kernel_launches(void);

/* Kernels that wait on on-chip barriers bound every wait (1 s); when one
 * expires the kernel records it in a per-device error word, stops and exits
 * cleanly.  This call synchronises `stream`, reads the word and returns
 * CSA_ERR_TIMEOUT if it is set (clearing it when `clear` is non-zero),
 * CSA_OK otherwise. */
csa_status_t csa_check_device_error(void* stream, int clear);

/*
 * Test hook for the launch-failure path (it never faults, traps or hangs a
 * GPU): the next kernel launch of any entry point is skipped, after its
 * arguments were validated, and the call returns CSA_ERR_CUDA for
 * `cuda_error` (a cudaError_t value > 0), as a failing launch would.  One
 * shot; process-wide.  cudaErrorNotSupported (801) is rejected with
 * CSA_ERR_INVALID_ARG: the packed entry points read that code from a launch
 * as "run one launch per sequence instead", so it would not surface.
 */
csa_status_t csa_debug_inject_launch_error(int cuda_error);

/*
 * Test hook for the timeout path (it never faults, traps or hangs a GPU).
 * `ns`: the time limit, in ns, of each bounded wait of the tensor-core
 * kernels' work in launches made after this call (0: back to the default
 * 1 s; < 0: CSA_ERR_INVALID_ARG).  `stall_next` != 0: the next tensor-core
 * launch (prefill indexer or attention) makes one thread of every CTA wait on
 * a barrier that nothing completes, so that wait runs out after `ns`.  When a
 * wait runs out the kernel records CSA_ERR_TIMEOUT in the device error word,
 * every CTA stops issuing work, waits (with the default limit) for the copies
 * and MMAs it already issued, releases its tensor memory and exits; outputs
 * of that launch are unspecified, later launches see the word set and do
 * nothing until csa_check_device_error clears it.  Process-wide.
 */
csa_status_t csa_debug_set_wait_limit(long long ns, int stall_next);

/*
 * csa_compress -- stage 1: overlapping (or plain) mean-pool compression
 * followed by a projection, optionally quantised to fp8.
 * Follows "百万上下文从「奢侈品」变「日用品」…" §3.2 (C[i] = W . mean of the
 * block's rows, floor(n/m) entries) and "DS-V4 分析&学习" §1.3 (2m-position
 * overlapping windows); ratio 128 without overlap per "DeepSeek V4 CSA + CP
 * 迁移到 HP…" §3.2.
 *
 *   out[b, i, :] = (mean_{p in win(i)} x[b, p, :]) @ W,   0 <= i < floor(n/m)
 *     overlap = 1: win(i) = [m(i-1), m(i+1)) ∩ [0, n)  (own block + previous)
 *     overlap = 0: win(i) = [m i, m(i+1))
 *
 *   x     [B, n, d_in]     x_dt = CSA_DT_F32 or CSA_DT_BF16
 *   W     [d_in, d_out]    same dtype as x, applied as row-vector @ W
 *   out   [B, floor(n/m), d_out]  out_dt:
 *           CSA_DT_F32  (x_dt F32 only), CSA_DT_BF16 (round to nearest even),
 *           CSA_DT_E4M3 (uint8 codes; out_row_scale [B, floor(n/m)] fp32 gets
 *           amax/448 of the row, 1 for a zero row; code = E4M3(v/scale),
 *           nearest-even, saturating)
 *           CSA_DT_E4M3_HADAMARD: as CSA_DT_E4M3, of the row rotated first by
 *           the normalised Walsh-Hadamard matrix H (d_out a power of two): in
 *           fp32, for stride s = 1, 2, ..., d_out/2 each pair (i, i+s) with
 *           i & s == 0 becomes (x_i + x_{i+s}, x_i - x_{i+s}), then every value
 *           is multiplied by fp32(1/sqrt(d_out)).  H is orthonormal, so
 *           indexer scores against rotated queries are unchanged up to the fp8
 *           rounding, which the rotation spreads over all channels (a reading
 *           of the DSA-lineage fp8 indexer that "DS-V4 分析&学习" §1.2 builds
 *           on; no formula for it is printed there).
 *   out_row_scale  required iff out_dt is an E4M3 type, else must be NULL.
 *   Limits: 16 <= d_in, d_out <= 256 and multiples of 16; m >= 1.
 *   Pooling and the projection accumulate in fp32.
 */
csa_status_t csa_compress(const void* x, int x_dt, int B, int n, int d_in, const void* W,
                          int d_out, int m, int overlap, void* out, int out_dt,
                          float* out_row_scale, void* stream);

/*
 * csa_compress_gated -- stage 1, learned variant: the gated-softmax
 * compressor.  "DeepSeek V4 CSA + CP 迁移到 HP：困难点深度分析" §3.2 lists the
 * production compressor's parts (a KV projection linear_wkv, a gate
 * projection linear_wgate, softmax / split / reshape, an APE parameter;
 * ratio 4 overlapping, ratio 128 not) without a formula; this is the reading:
 *
 *   c = 2 if overlap else 1;  for every position p:
 *     v_p = x[b, p] @ W_kv,   z_p = x[b, p] @ W_gate + ape[p mod m]   (c*d_out each)
 *   entry i < floor(n/m), channel e < d_out:
 *     overlap: terms (z_p[e], v_p[e]) for p in block i-1 (absent for i = 0)
 *              and (z_p[d_out+e], v_p[d_out+e]) for p in block i;
 *     plain:   terms (z_p[e], v_p[e]) for p in block i;
 *     out[b, i, e] = sum_terms softmax(z) v.
 *
 *   x      [B, n, d_in]       x_dt CSA_DT_F32 or CSA_DT_BF16
 *   W_kv, W_gate [d_in, c*d_out]  same dtype as x
 *   ape    [m, c*d_out]       fp32
 *   out, out_dt, out_row_scale: as csa_compress (fp32 / bf16 / E4M3 / rotated E4M3).
 *   Limits: 16 <= d_in, d_out <= 256, multiples of 16; m >= 1.  Projections,
 *   softmax and pooling run in fp32 (expf).
 *   Errors as csa_compress; nothing is launched on a validation error.
 */
csa_status_t csa_compress_gated(const void* x, int x_dt, int B, int n, int d_in, const void* W_kv,
                                const void* W_gate, const float* ape, int d_out, int m, int overlap,
                                void* out, int out_dt, float* out_row_scale, void* stream);

/*
 * csa_compress_append -- decode-time stage 1: one new token per batch element
 * updates the compressor state and, when it completes a block, writes that
 * block's compressed entry into the cache.
 * Follows "DS-V4 分析&学习", opening summary (the KV cache is the compressed
 * cache plus a state cache and a tail state) and §1.3 (an overlapping entry
 * spans the previous and the current block, so decode keeps both sums).
 *
 *   state[b, 0, :]  sum of the last complete block's m rows        (fp32)
 *   state[b, 1, :]  running sum of the current block                (fp32)
 *   For the token at absolute position p = pos[b] (p < 0: element b has no
 *   token this step and nothing of it changes):
 *     state[b, 1, :] += x_new[b, :]
 *     if (p + 1) % m == 0, block j = p / m is complete:
 *       cache[b, j, :] = (mean of blocks j-1 and j if overlap and j > 0,
 *                         else of block j alone) @ W       (if j < N_cap)
 *       n_entries[b] = j + 1                   (if j < N_cap and n_entries != NULL)
 *       state[b, 0, :] = state[b, 1, :];  state[b, 1, :] = 0
 *   Feeding positions 0 .. n-1 in order reproduces csa_compress on the whole
 *   sequence (up to fp32 rounding of the sums).
 *
 *   x_new  [B, d_in]        x_dt = CSA_DT_F32 or CSA_DT_BF16
 *   W      [d_in, d_out]    same dtype as x_new
 *   pos    device int32 [B]
 *   state  device fp32 [B, 2, d_in], caller-owned, zero before the first token
 *   cache  [B, N_cap, d_out]  out_dt as in csa_compress (E4M3 types:
 *          cache_scale [B, N_cap] fp32 gets the row's amax/448; the Hadamard
 *          type rotates the row first); cache_scale required iff out_dt is an
 *          E4M3 type, else NULL.
 *   n_entries  device int32 [B] or NULL.
 *   Limits as csa_compress.  Calls on one state must be ordered (same stream
 *   or synchronised): each call reads and writes it.
 */
csa_status_t csa_compress_append(const void* x_new, int x_dt, int B, int d_in, const void* W,
                                 int d_out, int m, int overlap, const int* pos, float* state,
                                 void* cache, int out_dt, float* cache_scale, int N_cap,
                                 int* n_entries, void* stream);

/*
 * csa_indexer_topk -- stage 2: Lightning-Indexer score + causal per-query
 * top-k, fused: the score matrix never reaches global memory.
 * Follows "百万上下文从「奢侈品」变「日用品」…" §3.2 (query . compressed-key
 * score, torch.topk per query) and §8.2 (scores must not be materialised),
 * "DS-V4 分析&学习" §1.2 and §4 (low-precision indexer QK).
 *
 *   score[t, s] = sum_h w[t, h] * ReLU(qI[t, h, :] . kI[s, :])  for visible s
 *   idx_out[b, q, :] = the topk entries of largest score; equal scores are
 *     taken lowest index first; with V < topk visible entries the row holds
 *     those V entries followed by -1.  The order inside a row is not part of
 *     the contract (it is deterministic).
 *
 *   qI [B, n_q, H_I, d_I]: qI_dt F32, BF16, or E4M3 with qI_scale [B, n_q, H_I].
 *      With kI_dt == CSA_DT_E4M3 and qI_dt == CSA_DT_BF16 (qI_scale NULL), each
 *      (query, head) row is quantised in the kernel exactly as csa_compress
 *      quantises a row (fp32: scale = amax/448, code = E4M3(x/scale)).
 *      With kI_dt == CSA_DT_E4M3_HADAMARD (keys from csa_compress with that
 *      type), a bf16 query row is rotated the same way before it is
 *      quantised; E4M3 query codes (qI_dt == CSA_DT_E4M3) are taken as given
 *      (already rotated).  Needs d_I a power of two; served by the fp8
 *      tensor-core and cluster kernels (d_I 64, or 128 for few rows).
 *   qI_weight [B, n_q, H_I] fp32: per-query, per-head gate weights w of any
 *      sign (the gated form of the DSA-lineage indexer that "DS-V4 分析&学习"
 *      §1.2 names; no formula is printed there), or NULL for w = 1.  Scores
 *      may then be negative; they still order as real numbers (-0 equals +0),
 *      below every zero score.  The weight multiplies the head's ReLU output,
 *      folded into the per-head query scale in fp32 by the kernels.
 *   kI [B, N_cap, d_I]: kI_dt F32, BF16, or E4M3 with kI_scale [B, N_cap].
 *      Supported pairs: (F32,F32), (BF16,BF16), (BF16,E4M3), (E4M3,E4M3).
 *      With fp8 the score is sk_s * sum_h sq_h * ReLU(q8_h . k8_s).
 *   n_entries [B] valid entries per element (NULL: N_cap); q_pos [B, n_q] (NULL: q).
 *   m: compression ratio (visibility rule above).  1 <= topk <= 2048.
 *   Limits: 1 <= H_I <= 16, d_I multiple of 16 and <= 256, N_cap <= 40960.
 *   idx_out [B, n_q, topk] int32.
 */
csa_status_t csa_indexer_topk(const void* qI, int qI_dt, const float* qI_scale,
                              const float* qI_weight, const void* kI,
                              int kI_dt, const float* kI_scale, int B, int n_q, int H_I, int d_I,
                              int N_cap, const int* n_entries, const int* q_pos, int m, int topk,
                              int* idx_out, void* stream);

/*
 * csa_sparse_attn -- stage 3: joint-softmax MQA over the selected compressed
 * entries plus the sliding window of raw KV (shared KV: one vector is both
 * key and value, one KV head for all query heads).
 * Follows "DS-V4 分析&学习" §1.2, §1.5 and "百万上下文从「奢侈品」变「日用品」…"
 * §5.2 (window [max(0,t-W+1), t], scale 1/sqrt(D)).
 *
 *   For query row (b, q) at position t and head h:
 *     keys = { kv_c[b, s] : s = idx[b, q, j], 0 <= s < N_cap }      (compressed)
 *          ∪ { kv_raw[b, j] : position raw_pos0[b]+j in [max(0,t-W+1), t] } (window)
 *     as a multiset (nothing de-duplicated), z = softmax_scale * q . key,
 *     out = sum softmax(z) key, lse_out = log(sum exp z) (natural log).
 *     An empty key set gives out = 0 and lse = -inf.
 *   q [B, n_q, H, D] and kv_c [B, N_cap, D], kv_raw [B, L_raw, D], out [B, n_q, H, D]
 *     share dt (CSA_DT_F32 or CSA_DT_BF16); accumulation is fp32.
 *   idx [B, n_q, topk] int32; negative entries are padding, entries >= N_cap
 *     are ignored.  topk may be 0 (window only; idx may then be NULL).
 *   raw_pos0 / raw_len [B] (NULL: 0 / L_raw); q_pos [B, n_q] (NULL: q).
 *   softmax_scale <= 0 selects 1/sqrt(D).  lse_out [B, n_q, H] fp32 or NULL.
 *   Limits: D multiple of 16, 16 <= D <= 256; H in {1,2,4,...,128}; window >= 0.
 */
csa_status_t csa_sparse_attn(const void* q, int dt, int B, int n_q, int H, int D,
                             const void* kv_c, int N_cap, const int* idx, int topk,
                             const void* kv_raw, int L_raw, const int* raw_pos0,
                             const int* raw_len, int window, const int* q_pos,
                             float softmax_scale, void* out, float* lse_out, void* stream);

/*
 * hca_dense_attn -- HCA: dense attention over every visible compressed entry
 * (no top-k) plus the sliding window, under one softmax.
 * Follows "DS-V4 分析&学习" §1.4 and "百万上下文从「奢侈品」变「日用品」…" §4.3.
 *
 *   keys = { kv_c[b, s] : s < min(floor((t+1)/m), n_entries[b], N_cap) } ∪ window,
 *   otherwise exactly as csa_sparse_attn.  n_entries [B] (NULL: N_cap).
 */
csa_status_t hca_dense_attn(const void* q, int dt, int B, int n_q, int H, int D,
                            const void* kv_c, int N_cap, const int* n_entries, int m,
                            const void* kv_raw, int L_raw, const int* raw_pos0,
                            const int* raw_len, int window, const int* q_pos,
                            float softmax_scale, void* out, float* lse_out, void* stream);

/*
 * Paged caches (serving layout).  The _paged entry points below take the
 * compressed caches as a pool of fixed-size pages instead of one [B, N_cap, *]
 * block per element:
 *   pool          [num_pages, page_size, row]   (kv_c rows, or indexer-key rows,
 *                 with the per-row fp32 scales as a pool [num_pages, page_size])
 *   block_table   device int32 [B, max_pages]: logical entry s of element b
 *                 lives at row s mod page_size of page block_table[b][s / page_size].
 *   page_size     a power of two in [1, 2^20]; the logical capacity is
 *                 N_cap = max_pages * page_size (at most 2^30).
 * A page id outside [0, num_pages) marks a page that is not there: its entries
 * are never read or written (attention skips them like padding, the indexer
 * scores them as zero rows, append drops the write).  Every other argument,
 * the arithmetic and the results are those of the unpaged entry point of the
 * same name; paged calls are served by the decode kernels (cluster-split and
 * SIMT), not the prefill tensor-core kernels.  These calls are this library's
 * serving layout, not a step the pages describe (they name paged KV pools for
 * serving, "百万上下文从「奢侈品」变「日用品」…" §8.3).
 */
csa_status_t csa_compress_append_paged(const void* x_new, int x_dt, int B, int d_in, const void* W,
                                       int d_out, int m, int overlap, const int* pos, float* state,
                                       void* cache_pages, int out_dt, float* cache_scale_pages,
                                       const int* block_table, int max_pages, int page_size,
                                       int num_pages, int* n_entries, void* stream);

csa_status_t csa_indexer_topk_paged(const void* qI, int qI_dt, const float* qI_scale,
                                    const float* qI_weight, const void* kI_pages, int kI_dt,
                                    const float* kI_scale_pages, const int* block_table,
                                    int max_pages, int page_size, int num_pages, int B, int n_q,
                                    int H_I, int d_I, const int* n_entries, const int* q_pos,
                                    int m, int topk, int* idx_out, void* stream);

csa_status_t csa_sparse_attn_paged(const void* q, int dt, int B, int n_q, int H, int D,
                                   const void* kv_c_pages, const int* block_table, int max_pages,
                                   int page_size, int num_pages, const int* idx, int topk,
                                   const void* kv_raw, int L_raw, const int* raw_pos0,
                                   const int* raw_len, int window, const int* q_pos,
                                   float softmax_scale, void* out, float* lse_out, void* stream);

csa_status_t hca_dense_attn_paged(const void* q, int dt, int B, int n_q, int H, int D,
                                  const void* kv_c_pages, const int* block_table, int max_pages,
                                  int page_size, int num_pages, const int* n_entries, int m,
                                  const void* kv_raw, int L_raw, const int* raw_pos0,
                                  const int* raw_len, int window, const int* q_pos,
                                  float softmax_scale, void* out, float* lse_out, void* stream);

/*
 * Packed (varlen) prefill.  S sequences are packed along the token dimension:
 * sequence s owns tokens [cu_seqlens[s], cu_seqlens[s+1]) (cu_seqlens: HOST
 * int32 [S+1], cu_seqlens[0] = 0, non-decreasing) and, in the packed
 * compressed dimension, entries [e(s), e(s+1)) with
 * e(s) = sum_{s' < s} floor(len(s') / m) (csa_varlen_entry_offsets).  Each
 * sequence is computed exactly as the unpacked call with B = 1, n = len(s)
 * would compute it: positions, the visibility rule, the window and the top-k
 * are local to the sequence, and indices in idx are entries of the sequence
 * (0 .. floor(len/m) - 1, -1 padding).  "DeepSeek V4 CSA + CP 迁移到 HP：
 * 困难点深度分析" names this layout: actual_seq_len in the attention's
 * construct signature (§4.2) and compressed cu_seqlens with packed-sequence
 * support in its migration plan (Phase 3).  The alignment rule applies to
 * every sequence's slice (it holds whenever the base pointers follow it,
 * since rows are multiples of 16 bytes).  All sequences are validated
 * before the first launch; the calls
 * launch one kernel per non-empty sequence (capturable in a CUDA graph).
 *   tensors: packed forms of the unpacked calls' arguments, e.g. for
 *   csa_sparse_attn_varlen q / out [T, H, D], kv_c [E, D], idx [T, topk],
 *   kv_raw [T, D], lse_out [T, H]; T = cu_seqlens[S], E = e(S).
 */
int csa_varlen_entry_offsets(const int* cu_seqlens, int S, int m, int* entry_offsets);
/*   writes e(0..S) into entry_offsets [S+1] (host) and returns e(S), or -1 on
 *   an invalid argument (S < 0, m < 1, NULL arrays, cu_seqlens[0] != 0 or a
 *   decreasing cu_seqlens). */

csa_status_t csa_compress_varlen(const void* x, int x_dt, int S, const int* cu_seqlens, int d_in,
                                 const void* W, int d_out, int m, int overlap, void* out,
                                 int out_dt, float* out_row_scale, void* stream);

csa_status_t csa_indexer_topk_varlen(const void* qI, int qI_dt, const float* qI_scale,
                                     const float* qI_weight, const void* kI, int kI_dt,
                                     const float* kI_scale, int S, const int* cu_seqlens, int H_I,
                                     int d_I, int m, int topk, int* idx_out, void* stream);

csa_status_t csa_sparse_attn_varlen(const void* q, int dt, int S, const int* cu_seqlens, int H,
                                    int D, const void* kv_c, int m, const int* idx, int topk,
                                    const void* kv_raw, int window, float softmax_scale, void* out,
                                    float* lse_out, void* stream);

csa_status_t hca_dense_attn_varlen(const void* q, int dt, int S, const int* cu_seqlens, int H,
                                   int D, const void* kv_c, int m, const void* kv_raw, int window,
                                   float softmax_scale, void* out, float* lse_out, void* stream);

/*
 * Query spans at an offset (context-parallel shards).  "DeepSeek V4 CSA + CP
 * 迁移到 HP：困难点深度分析" lays a long sequence over ranks (the pipeline that
 * opens the page): a rank holds spans of consecutive positions, all-gathers
 * the compressed entries and runs stage 2 and 3 for its own queries, whose
 * positions start past 0.  These calls are the unpacked calls with q_pos and
 * raw_pos0 / raw_len given as uniform host offsets:
 *   query q of every element sits at position q_pos0 + q (q_pos0 >= 0);
 *   raw row j of every element holds position raw_pos0 + j (raw_pos0 >= 0),
 *   all L_raw rows present (raw_len = L_raw).
 * Every other argument, the arithmetic, the error behaviour and the results
 * are those of csa_indexer_topk / csa_sparse_attn / hca_dense_attn with
 * q_pos[b][q] = q_pos0 + q, raw_pos0[b] = raw_pos0 and raw_len[b] = L_raw.
 * Unlike a per-element position array, a uniform offset keeps the prefill
 * shape, so these calls take the tensor-core kernels (64 heads x 128, d_I 64)
 * where the unpacked prefill call would.
 */
csa_status_t csa_indexer_topk_at(const void* qI, int qI_dt, const float* qI_scale,
                                 const float* qI_weight, const void* kI, int kI_dt,
                                 const float* kI_scale, int B, int n_q, int H_I, int d_I,
                                 int N_cap, const int* n_entries, int q_pos0, int m, int topk,
                                 int* idx_out, void* stream);

csa_status_t csa_sparse_attn_at(const void* q, int dt, int B, int n_q, int H, int D,
                                const void* kv_c, int N_cap, const int* idx, int topk,
                                const void* kv_raw, int L_raw, int raw_pos0, int window,
                                int q_pos0, float softmax_scale, void* out, float* lse_out,
                                void* stream);

csa_status_t hca_dense_attn_at(const void* q, int dt, int B, int n_q, int H, int D,
                               const void* kv_c, int N_cap, const int* n_entries, int m,
                               const void* kv_raw, int L_raw, int raw_pos0, int window,
                               int q_pos0, float softmax_scale, void* out, float* lse_out,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_B200_H */
