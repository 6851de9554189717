/*
 * waveprune.h — C ABI of libwaveprune.so: WavePrune causal attention on
 * NVIDIA B200 (sm_100a).
 *
 * WavePrune keeps each RoPE channel's contribution to a query-key logit only
 * while the query-key distance is within one period of that channel, and adds
 * 0 (not -inf) otherwise. Pages cited below, by title:
 *   [RN] "WavePrune：RoPE 通常只需一个旋转周期" — reading notes of
 *        arXiv:2610.06963 "WavePrune: One period is often enough for RoPE".
 *   [KC] "WavePrune：RoPE只用一个旋转周期，长文本性能反而更好".
 *   [TW] "Guancheng Du @ducatiqwq" — the author's thread.
 *
 * Conventions for every call:
 *   - Return value is a wp_status. Argument checks run on the host before any
 *     launch; a failing check launches nothing. Launch failures give
 *     WP_ERR_CUDA. Nothing in the library exits or aborts the process.
 *   - Device pointers must be 16-byte aligned and tensors contiguous in the
 *     stated layout. The caller owns every buffer and the stream; the library
 *     allocates no device memory. Device calls are asynchronous on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - A kernel that waits longer than the wait limit on one of its internal
 *     barriers stops, records WP_ERR_TIMEOUT in a device status word and
 *     returns; wp_device_status() reads and clears that word. The word
 *     carries over between calls: while it is set, every wp_prefill on that
 *     device skips its work and writes NaN to all its O rows and LSE entries
 *     (the call itself still returns WP_OK), until wp_device_status() has
 *     read and cleared it. Outputs are never left holding stale values.
 *   - bf16 is IEEE bfloat16 (raw 16-bit patterns); outputs round to nearest
 *     even.
 */
#ifndef WAVEPRUNE_H
#define WAVEPRUNE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WP_OK = 0,
    WP_ERR_ARG = 1,          /* invalid argument (NULL, size, alignment, value) */
    WP_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d_h not 64/128) */
    WP_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
    WP_ERR_TIMEOUT = 4       /* a kernel gave up waiting on an internal barrier */
} wp_status;

/* RoPE rotation layouts. Interleaved [KC, RoPE matrix]: channel c rotates the
 * dim pair (2c, 2c+1). Half-split: channel c rotates (c, c + d_h/2), the
 * rotate_half convention of Llama/Qwen checkpoints.
 * WP_ROPE_HALF_SPLIT_PAIRED is for wp_rope_apply only: it rotates a half-split
 * input exactly as WP_ROPE_HALF_SPLIT and writes channel c's pair to dims
 * (2c, 2c+1) of the output, i.e. in the interleaved order. Q.K^T is unchanged
 * when Q and K are permuted alike (V is untouched), so attention on paired Q
 * and K is attention on the half-split model; wp_cutoffs, wp_prefill and
 * wp_decode then take WP_ROPE_INTERLEAVED, and every 16-dim group holds 8
 * whole channels: the group-end cutoffs of [RN §2.3, Table 12]
 * (28, 160, 900, 5063, ... at theta 1e6) instead of the half-split groups'
 * max over channels c and c + d_h/2. */
enum { WP_ROPE_INTERLEAVED = 0, WP_ROPE_HALF_SPLIT = 1, WP_ROPE_HALF_SPLIT_PAIRED = 2 };

/* Logit modes. Channel mode is the exact per-channel rule [RN §2.1, Eq. (6)];
 * grouped mode gives each 16-dim group the largest cutoff of the channels
 * owning its dims [RN §2.3, Eq. (8); TW (6/7)]. */
enum { WP_MODE_GROUPED = 0, WP_MODE_CHANNEL = 1 };

/* A cutoff that never masks. */
#define WP_CUTOFF_INF INT32_MAX

/* Tile classes written by wp_schedule. */
enum { WP_TILE_SKIP = 0, WP_TILE_FULL = 1, WP_TILE_BOUNDARY = 2, WP_TILE_NONE = 3 };

/*
 * wp_cutoffs — integer cutoff tables, host only, fp64.
 * [RN §1.1, Eq. (2)-(5)]: f_c = theta^(-2c/d_h), c = 0..d_h/2-1, times any
 * frequency scale (the cutoffs follow the scaled frequencies, [RN §1.1]).
 * [RN §2.1, after Eq. (6)]: w_c = alpha*pi/f_c (alpha = 2: one period) and a
 * channel is kept iff distance <= floor(w_c). [RN §2.3, Eq. (8)]: the cutoff of
 * group g (dims [16g, 16g+16)) is the max over the channels owning its dims.
 *   d_h          head dim, a multiple of 16 (>= 16).
 *   theta        RoPE base, > 1.
 *   freq_scale   host [d_h/2] per-channel multipliers of f_c, or NULL (= 1).
 *   scale_all    uniform multiplier of f_c (e.g. 0.25 = position interpolation
 *                by 4), finite and > 0.
 *   alpha        period multiple, > 0 (2.0 = the pages' default).
 *   layout       WP_ROPE_INTERLEAVED or WP_ROPE_HALF_SPLIT.
 *   chan_cut     host out [d_h/2] (may be NULL); group_cut host out [d_h/16]
 *                (may be NULL). Values saturate at WP_CUTOFF_INF.
 * Touches no GPU. Errors: WP_ERR_ARG.
 */
int wp_cutoffs(int d_h, double theta, const double *freq_scale, double scale_all, double alpha, int layout,
               int32_t *chan_cut, int32_t *group_cut);

/*
 * wp_rope_apply — rotate bf16 Q or K by position * f_c [KC, RoPE matrix;
 * RN §1.1: the channel at position i rotates by i*f_c].
 *   x, y        device bf16 [B, N, H, d_h]; y may equal x (in place), other
 *               overlap is not allowed.
 *   pos         device int32 [B, N] positions, or NULL: position = pos0 + t.
 *   theta, freq_scale (host, [d_h/2] or NULL), scale_all, layout: as in
 *               wp_cutoffs; frequencies are formed in fp64 on the host.
 *   layout      also WP_ROPE_HALF_SPLIT_PAIRED (see its enum); then y must not
 *               overlap x at all (WP_ERR_ARG).
 * The angle is formed and reduced modulo 2*pi in fp64, the rotation is fp32,
 * the result rounds to bf16. d_h in {64, 128}. Errors: WP_ERR_ARG,
 * WP_ERR_UNSUPPORTED, WP_ERR_CUDA.
 */
int wp_rope_apply(const void *x, void *y, int B, int N, int H, int d_h, const int32_t *pos, int pos0, double theta,
                  const double *freq_scale, double scale_all, int layout, void *stream);

/*
 * wp_schedule — tile classes of a causal (query block, key block) grid, host
 * only [RN §2.3, the three-row table; TW (6/7)]. For a tile holding at least
 * one pair j <= i, the distances span [dmin, dmax]; a cutoff W marks the tile
 * WP_TILE_SKIP if dmin > W, WP_TILE_FULL if dmax <= W, WP_TILE_BOUNDARY
 * otherwise. Tiles with no causal pair are WP_TILE_NONE and not counted.
 * The prefill kernel classifies its tiles with this same function.
 *   N, BM, BN   sequence length and block sizes (> 0).
 *   cut         host [n_cut] cutoffs (>= 0), n_cut in 1..64.
 *   cls         host out [nqb][nkb][n_cut] uint8 (nqb = ceil(N/BM),
 *               nkb = ceil(N/BN)), or NULL.
 *   counts      host out [n_cut][3] int64: skip, full, boundary.
 * Errors: WP_ERR_ARG.
 */
int wp_schedule(int N, int BM, int BN, const int32_t *cut, int n_cut, uint8_t *cls, int64_t *counts);

/*
 * wp_prefill — causal WavePrune attention over positions 0..N-1, so that the
 * distance of a pair is i - j [RN §2.1, Eq. (6) and the softmax after it].
 *   q           device bf16 [B, N, H_q, d_h], rotated.
 *   k, v        device bf16 [B, N, H_kv, d_h], k rotated. H_q % H_kv == 0;
 *               query head h reads KV head h / (H_q / H_kv).
 *   o           device bf16 out [B, N, H_q, d_h].
 *   lse         device fp32 out [B, H_q, N]: natural-log logsumexp of the
 *               row's logits (softmax scale included), or NULL.
 *   mode        WP_MODE_GROUPED: cut = host group_cut [d_h/16] — the fast path
 *               (TMA loads of only the K columns of non-skipped groups, one
 *               tcgen05 MMA per 16-dim group into TMEM; on a tile where a
 *               group is partly in window its contribution is masked per
 *               element in the logit tile before the remaining groups add in).
 *               WP_MODE_CHANNEL: cut = host chan_cut [d_h/2] — exact rule,
 *               correctness path (CUDA cores), not tuned for speed.
 *               cut = NULL means every cutoff is WP_CUTOFF_INF (dense).
 *   layout      rotation layout; used by channel mode to pair dims.
 *   softmax_scale  > 0, or <= 0 for 1/sqrt(d_h) [RN §2.1, detail 3].
 * d_h in {64, 128}. Masked channels add 0 to the logit (the pair still takes
 * part in the softmax) [RN §2.1, detail 1]. Errors: WP_ERR_ARG,
 * WP_ERR_UNSUPPORTED (also: B*H_kv above 65535; grouped mode with N above
 * 2^20, the longest sequence whose key-block table fits one CTA's shared
 * memory), WP_ERR_CUDA.
 */
int wp_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B, int N, int H_q, int H_kv,
               int d_h, int mode, const int32_t *cut, int layout, float softmax_scale, void *stream);

/*
 * wp_prefill_ex — wp_prefill with one cutoff table per query head, and
 * packed batches of sequences of different lengths. [RN §5] names
 * head-specific thresholds as the next step after one table per model; the
 * rule per head is the same as in wp_prefill.
 *   cu_seqlens  NULL: a uniform batch, laid out as in wp_prefill (q, o
 *               [B, N, H_q, d_h]; k, v [B, N, H_kv, d_h]; lse [B, H_q, N]);
 *               total_tokens is ignored.
 *               Otherwise device int32 [B+1], 4-byte aligned: sequence b is
 *               rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of the packed
 *               q, o [T, H_q, d_h] and k, v [T, H_kv, d_h] (T = total_tokens),
 *               positions restart at 0 in every sequence, and lse is
 *               [H_q, T]. N is an upper bound of the lengths (it sizes the
 *               launch). A sequence whose offsets fall outside [0, T], run
 *               backwards, or span more than N rows is skipped (its rows are
 *               not written) and WP_ERR_ARG is recorded in the device status
 *               word (see wp_device_status). Rows past the end of a sequence
 *               are read only where the causal mask gives them weight exactly
 *               0; V must therefore be finite in the whole buffer.
 *   cut, cut_rows  cut_rows = 1: one table for every head (as in wp_prefill);
 *               cut_rows = H_q: cut is [H_q][d_h/16] (grouped) or
 *               [H_q][d_h/2] (channel mode), row h for query head h (two
 *               heads that share a KV head share its K loads, which cover the
 *               groups either of them keeps). cut may be NULL only with
 *               cut_rows = 1 (dense).
 * Everything else as in wp_prefill. Errors: those of wp_prefill, and
 * WP_ERR_ARG (cut_rows not 1 or H_q; cu_seqlens misaligned or
 * total_tokens <= 0 with cu_seqlens), WP_ERR_UNSUPPORTED (more than 2048
 * table entries in all, i.e. cut_rows x d_h/16 or cut_rows x d_h/2;
 * total_tokens of 2^31 - 256 or more; grouped mode with cut_rows = H_q and N
 * above 2^19, where the two heads' key-block tables no longer fit one CTA's
 * shared memory).
 */
int wp_prefill_ex(const void *q, const void *k, const void *v, void *o, float *lse, const int32_t *cu_seqlens,
                  int B, int N, int64_t total_tokens, int H_q, int H_kv, int d_h, int mode, const int32_t *cut,
                  int cut_rows, int layout, float softmax_scale, void *stream);

/*
 * wp_prefill_backward_workspace_bytes — size of the scratch that
 * wp_prefill_backward needs (one fp32 per query row and head).
 */
size_t wp_prefill_backward_workspace_bytes(int B, int N, int H_q);

/*
 * wp_prefill_backward — gradients of a grouped-mode wp_prefill: given dO, the
 * gradients dQ, dK, dV of sum(dO * O) with respect to its inputs q (rotated),
 * k (rotated) and v. [RN §2.3, the paragraph on the backward kernel]: in the
 * backward the head dimension is the output axis of the dQ and dK products,
 * so the group mask is applied to the gradient operand dS = P * (dP - D)
 * before each product (full groups take dS as it is, skipped groups add
 * nothing), and dQ and dK come from the same masked operands; [RN §4.6,
 * Table 4] reports that the backward gains little. The pages print no
 * backward equations: this is the chain rule through wp_prefill's definition,
 *   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . V_j - D_i),  D_i = dO_i . O_i,
 *   dQ_i[g] = scale sum_j 1[i-j <= W_g] dS_ij K_j[g],
 *   dK_j[g] = scale sum_i 1[i-j <= W_g] dS_ij Q_i[g].
 *   q, o, dout  device bf16 [B, N, H_q, d_h]: the forward's inputs q, its
 *               output o and the incoming gradient.
 *   k, v        device bf16 [B, N, H_kv, d_h].
 *   lse         device fp32 [B, H_q, N]: the forward's LSE (natural log).
 *   dq          device bf16 out [B, N, H_q, d_h]; dk, dv device bf16 out
 *               [B, N, H_kv, d_h] (the query heads sharing a KV head add up).
 *   workspace   device scratch of at least
 *               wp_prefill_backward_workspace_bytes(B, N, H_q) bytes, 256-byte
 *               aligned (holds D).
 *   cut, cut_rows  group cutoffs as in wp_prefill_ex: cut_rows = 1 (cut
 *               [d_h/16], or NULL: dense) or H_q ([H_q][d_h/16]).
 *   softmax_scale  the forward's scale (<= 0: 1/sqrt(d_h)).
 * Grouped mode only. The products run on the tcgen05 tensor cores with bf16
 * operands (P and dS rounded to bf16) and fp32 accumulation in TMEM. The
 * status word (wp_device_status) works as for wp_prefill: a wait that gives
 * up records WP_ERR_TIMEOUT and the affected rows of dq, dk, dv are NaN.
 * d_h in {64, 128}. Errors: WP_ERR_ARG, WP_ERR_UNSUPPORTED (also: more than
 * 2048 table entries; more than 64 query heads per KV head; N above
 * 128 * 65535), WP_ERR_CUDA.
 */
int wp_prefill_backward(const void *q, const void *k, const void *v, const void *o, const void *dout, const float *lse,
                        void *dq, void *dk, void *dv, void *workspace, size_t ws_bytes, int B, int N, int H_q,
                        int H_kv, int d_h, const int32_t *cut, int cut_rows, float softmax_scale, void *stream);

/*
 * wp_decode_workspace_bytes — size of the scratch that wp_decode needs for
 * the split-KV partial results of a batch (fp32 partial O and LSE per split).
 */
size_t wp_decode_workspace_bytes(int B, int H_q, int d_h, int Lmax);

/*
 * wp_decode — one new query per sequence against a KV cache, grouped cutoffs.
 * The query sits at position lens[b]-1 and attends keys 0..lens[b]-1, key j at
 * distance lens[b]-1-j. [RN §2.3, table row 1]: in decode a skipped group's
 * K bytes are not read; V is read in full.
 *   q           device bf16 [B, H_q, d_h], rotated.
 *   kcache, vcache  device bf16 [B, H_kv, Lmax, d_h] (keys rotated).
 *   lens        device int32 [B], each in 1..Lmax (a length outside that
 *               range makes the kernel write NaN rows for that sequence).
 *   group_cut   host [d_h/16] (NULL: dense).
 *   o           device bf16 out [B, H_q, d_h]; lse device fp32 out [B, H_q]
 *               or NULL.
 *   workspace   device scratch of at least wp_decode_workspace_bytes(...)
 *               bytes, 256-byte aligned; contents on entry do not matter.
 * Split-KV: the cache is streamed in key chunks with 16-byte vector loads;
 * each chunk's partial (O, LSE) is merged by LSE. d_h in {64, 128}.
 * Errors: WP_ERR_ARG, WP_ERR_UNSUPPORTED, WP_ERR_CUDA.
 */
int wp_decode(const void *q, const void *kcache, const void *vcache, const int32_t *lens, int Lmax, int B, int H_q,
              int H_kv, int d_h, const int32_t *group_cut, float softmax_scale, void *o, float *lse,
              void *workspace, size_t ws_bytes, void *stream);

/*
 * K cache layouts of wp_decode_kl.
 *   WP_KCACHE_ROWS          [B, H_kv, Lmax, d_h]: one row of d_h per key (the
 *                           layout of wp_decode).
 *   WP_KCACHE_GROUP_MAJOR   [B, H_kv, d_h/16, Lmax, 16]: the 16 dims of group g
 *                           of all keys are contiguous 32-byte records. [RN
 *                           §2.3, table row 1] says a skipped group's K bytes
 *                           are not read in decode; in this layout the keys a
 *                           group skips are one contiguous range, which DRAM
 *                           then never moves (in rows they are 32-byte holes
 *                           inside 256-byte rows that travel with their line).
 *                           The pages fix no layout; this one is a choice of
 *                           this library.
 */
enum wp_kcache_layout { WP_KCACHE_ROWS = 0, WP_KCACHE_GROUP_MAJOR = 1, WP_KCACHE_WINDOWED = 2 };

/*
 * WP_KCACHE_WINDOWED — the K cache with every group's out-of-window keys
 * evicted (KV eviction at the granularity the kernels read: a 16-dim group,
 * not a single channel). [RN §2.3, last paragraph] leaves freeing cache
 * capacity as future work; a decode at position len - 1 reads group g only
 * for keys j >= len - 1 - W_g, and len only grows, so a key older than W_g
 * positions is never read for that group again. Layout, per (b, hk): the
 * groups' rings back to back; group g keeps cap_g = min(round_up_16(W_g + 1),
 * round_up_16(Lmax)) records of 16 bf16, key j in slot j mod cap_g. Its size
 * per (b, hk) is wp_kcache_windowed_elems(Lmax, d_h, group_cut) elements;
 * the 32K decode workload's half-split table keeps 54 % of the K cache.
 * Decode it with wp_decode_kl(k_layout = WP_KCACHE_WINDOWED) and the SAME
 * group_cut it was built with (the table fixes the geometry; a different
 * table reads the wrong slots). Grouped mode, shared table, contiguous
 * cache only.
 */

/* Elements (bf16) of one (b, hk) of a windowed K cache; 0 on bad arguments. */
size_t wp_kcache_windowed_elems(int Lmax, int d_h, const int32_t *group_cut);

/*
 * wp_kcache_windowed_from_rows — build a windowed K cache from rows.
 *   k_rows    device bf16 [B, H_kv, Lmax, d_h] (read only), 16-byte aligned.
 *   lens      device int32 [B]: keys 0 .. lens[b]-1 are the sequence's.
 *   k_win     device bf16 out, B * H_kv * wp_kcache_windowed_elems(...)
 *             elements, 16-byte aligned, not overlapping k_rows; slot s of
 *             group g receives the latest key j < lens[b] with j mod cap_g = s
 *             (zeros where there is none).
 *   group_cut the group cutoffs [d_h/16] (required).
 * Asynchronous on `stream`. Errors: WP_ERR_ARG, WP_ERR_UNSUPPORTED (d_h),
 * WP_ERR_CUDA.
 */
int wp_kcache_windowed_from_rows(const void *k_rows, const int32_t *lens, void *k_win, int B, int H_kv, int Lmax,
                                 int d_h, const int32_t *group_cut, void *stream);

/*
 * wp_kcache_windowed_append — write one new key per sequence into a windowed
 * K cache: k_new device bf16 [B, H_kv, d_h] (the token at position pos[b],
 * device int32 [B]) into slot pos[b] mod cap_g of every group. A position
 * outside [0, Lmax) writes nothing. Errors as wp_kcache_windowed_from_rows.
 */
int wp_kcache_windowed_append(const void *k_new, const int32_t *pos, void *k_win, int B, int H_kv, int Lmax, int d_h,
                              const int32_t *group_cut, void *stream);

/*
 * wp_kcache_group_major — copy a K cache from WP_KCACHE_ROWS to
 * WP_KCACHE_GROUP_MAJOR.
 *   k_rows  device bf16 [B, H_kv, Lmax, d_h], 16-byte aligned (read only).
 *   k_gm    device bf16 out [B, H_kv, d_h/16, Lmax, 16], 16-byte aligned, the
 *           same size, caller-owned, not overlapping k_rows.
 *   d_h in {64, 128}. Asynchronous on `stream`.
 * Errors: WP_ERR_ARG (null, misaligned, same buffer, bad sizes),
 * WP_ERR_UNSUPPORTED (d_h), WP_ERR_CUDA.
 */
int wp_kcache_group_major(const void *k_rows, void *k_gm, int B, int H_kv, int Lmax, int d_h, void *stream);

/*
 * wp_decode_kl — wp_decode with the K cache in layout `k_layout`
 * (wp_kcache_layout); V stays [B, H_kv, Lmax, d_h]. All other arguments,
 * results and errors are those of wp_decode; a k_layout outside the enum is
 * WP_ERR_ARG. All layouts give bit-identical results. WP_KCACHE_WINDOWED
 * needs group_cut (WP_ERR_ARG without) and is WP_ERR_UNSUPPORTED in
 * wp_decode_ex's masked modes and in wp_decode_paged.
 */
int wp_decode_kl(const void *q, const void *kcache, int k_layout, const void *vcache, const int32_t *lens, int Lmax,
                 int B, int H_q, int H_kv, int d_h, const int32_t *group_cut, float softmax_scale, void *o, float *lse,
                 void *workspace, size_t ws_bytes, void *stream);

/*
 * wp_decode_ex — wp_decode_kl with the exact per-channel rule or one cutoff
 * table per query head.
 *   mode, cut, cut_rows, layout:
 *     WP_MODE_GROUPED, cut_rows = 1: cut is group_cut [d_h/16] (as wp_decode).
 *     WP_MODE_GROUPED, cut_rows = H_q: cut is [H_q][d_h/16], row h for query
 *       head h ([RN §5]: head-specific thresholds). The K loads cover the
 *       union of the heads' windows; each head's scores keep a group's
 *       product only while the key is in that head's window.
 *     WP_MODE_CHANNEL, cut_rows = 1: cut is chan_cut [d_h/2] (NULL: dense),
 *       the exact rule of [RN §2.1, Eq. (6)]; layout (WP_ROPE_INTERLEAVED or
 *       WP_ROPE_HALF_SPLIT) says which channel owns a dim. The decode query
 *       has one position, so the dims of a channel out of window are zeroed
 *       per key before the product; a group's K bytes are skipped beyond its
 *       largest channel cutoff.
 *     WP_MODE_CHANNEL, cut_rows = H_q: cut is [H_q][d_h/2], row h the
 *       channel cutoffs of query head h, the exact rule per head. The query
 *       heads of a KV head share its K loads (a group's K bytes are skipped
 *       beyond the largest cutoff of its channels over all heads) and each
 *       head's product takes the K dims masked by its own row: one product
 *       per query head instead of one per KV head.
 * Everything else as in wp_decode_kl. Errors: those of wp_decode_kl, and
 * WP_ERR_ARG (mode, layout or cut_rows out of range, NULL cut with
 * cut_rows = H_q, a negative cutoff), WP_ERR_UNSUPPORTED (grouped mode with
 * H_q x d_h/16 above 1024; channel mode with cut_rows = H_q and H_q x d_h/2
 * above 2048).
 */
int wp_decode_ex(const void *q, const void *kcache, int k_layout, const void *vcache, const int32_t *lens, int Lmax,
                 int B, int H_q, int H_kv, int d_h, int mode, const int32_t *cut, int cut_rows, int layout,
                 float softmax_scale, void *o, float *lse, void *workspace, size_t ws_bytes, void *stream);

/*
 * wp_decode_paged — wp_decode_kl over a paged KV cache, as serving engines
 * keep it: the keys of a sequence live in fixed-size pages from a shared pool,
 * listed per sequence in a block table. (The pages' decode reads one
 * contiguous cache; paging only changes where each key block is read from.)
 *   k_pages     device bf16 K pool of n_pages pages, each [H_kv, page_size,
 *               d_h] in WP_KCACHE_ROWS or [H_kv, d_h/16, page_size, 16] in
 *               WP_KCACHE_GROUP_MAJOR (k_layout).
 *   v_pages     device bf16 V pool of n_pages pages, each [H_kv, page_size, d_h].
 *   page_size   keys per page, a multiple of 16 (>= 16).
 *   block_table device int32 [B, max_pages]: entry j of sequence b is the page
 *               holding its keys [j*page_size, (j+1)*page_size); only the
 *               entries below ceil(lens[b] / page_size) are read. An entry
 *               read outside [0, n_pages) makes the kernel write NaN rows for
 *               that sequence (nothing is read from it).
 *   lens        device int32 [B], each in 1..max_pages*page_size.
 *   workspace   at least wp_decode_workspace_bytes(B, H_q, d_h,
 *               max_pages*page_size) bytes, 256-byte aligned.
 * Everything else as in wp_decode; results are bit-identical to wp_decode_kl
 * on the same keys stored contiguously. Errors: WP_ERR_ARG (also: block_table
 * NULL or not 4-byte aligned, n_pages/max_pages < 1, page_size not a positive
 * multiple of 16), WP_ERR_UNSUPPORTED (also: max_pages*page_size > 2^30),
 * WP_ERR_CUDA.
 */
int wp_decode_paged(const void *q, const void *k_pages, int k_layout, const void *v_pages, int n_pages, int page_size,
                    const int32_t *block_table, int max_pages, const int32_t *lens, int B, int H_q, int H_kv, int d_h,
                    const int32_t *group_cut, float softmax_scale, void *o, float *lse, void *workspace,
                    size_t ws_bytes, void *stream);

/*
 * wp_decode_static — wp_decode without a workspace argument, for callers that
 * cannot allocate device memory (for example a serving engine whose device
 * memory is planned up front and handed out by its own pool, or a decode loop
 * that must never reach cudaMalloc/cudaFree, which can synchronise the
 * device). It allocates nothing: the split-KV partial results go to a
 * fixed-size scratch array of WP_DECODE_STATIC_SCRATCH_BYTES (16 MiB) that is
 * part of this library's device image, so every GPU that loads the library
 * holds it until the process exits. The pages have no counterpart of this
 * call; it is an interface for those callers.
 *   Arguments, layouts and results are those of wp_decode.
 *   The first call on a device looks up the scratch array's device address
 *   (once per device, with that device current); make that first call before
 *   any stream capture.
 *   Every call on a device shares the one array and leaves its contents
 *   behind; nothing in it needs to start at zero. Calls whose kernels overlap
 *   on the GPU (e.g. on two streams without ordering) race on the array.
 *   Errors: WP_ERR_ARG for a null or misaligned q, kcache, vcache, lens, o
 *   or lse (checked first, whatever the sizes); WP_ERR_UNSUPPORTED when
 *   wp_decode_workspace_bytes(B, H_q, d_h, Lmax) exceeds
 *   WP_DECODE_STATIC_SCRATCH_BYTES, or on a device ordinal of 64 or more
 *   (nothing is launched); otherwise those of wp_decode.
 */
#define WP_DECODE_STATIC_SCRATCH_BYTES (16u << 20)
int wp_decode_static(const void *q, const void *kcache, const void *vcache, const int32_t *lens, int Lmax, int B,
                     int H_q, int H_kv, int d_h, const int32_t *group_cut, float softmax_scale, void *o, float *lse,
                     void *stream);

/*
 * wp_device_status — synchronises `stream`, then reads and clears the device
 * status word of the current device. Returns WP_OK, WP_ERR_TIMEOUT (a kernel
 * gave up waiting since the last call), WP_ERR_ARG (a packed prefill met
 * out-of-range cu_seqlens) or WP_ERR_CUDA.
 */
int wp_device_status(void *stream);

/* wp_set_wait_limit — cycles a kernel waits on one internal barrier before it
 * gives up (default 2e9, about one second). Values <= 0 restore the default.
 * Returns the previous value. Host only. */
long long wp_set_wait_limit(long long cycles);

/* wp_wait_probe — launches one CTA that waits on a barrier nothing ever
 * completes, under the current wait limit; the kernel then records
 * WP_ERR_TIMEOUT and returns. Used to test the timeout path without faulting
 * or hanging the GPU. Errors: WP_ERR_CUDA. */
int wp_wait_probe(void *stream);

/* wp_status_str — static description of a status code. */
const char *wp_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* WAVEPRUNE_H */
