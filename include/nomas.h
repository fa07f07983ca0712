/*
 * nomas.h -- C ABI of libnomas: action-aware segment-causal attention over an
 * INT8 key/value cache with a sliding history window, for one NVIDIA B200
 * (sm_100a).
 *
 * The operations follow the Hy-Nomas pages (no API is given there; these
 * signatures are this library's statement of the problem):
 *   - fluxbbs.com "Hy-Nomas 拆解", section 架构: segment-causal attention
 *     (bidirectional inside a segment, a segment sees only itself and earlier
 *     segments, text and video K/V cached for the next segment) and the
 *     action-aware mask (one description head per segment visible across
 *     segments, action tails visible only in their own segment and time
 *     window);
 *   - same page, section 单卡 4090 怎么做到的: K/V stored as INT8 with float
 *     scale factors and dequantised to BF16 for compute; retained history
 *     limited to 18 latent frames; block-sparse attention keeping 25 % of the
 *     candidate video blocks after the first two denoising steps;
 *   - hyphentech.top, config table: at most 18 history latent frames on the
 *     GPU in the single-GPU setting, full history in the standard one.
 *
 * Conventions shared by every call
 *   - Ownership: the caller allocates every device buffer (sizes come from the
 *     *_bytes / *_layout queries).  The library allocates no device memory
 *     and never synchronises a stream, except nomas_device_status.
 *   - Pointers: device pointers, 16-byte aligned; bf16 tensors are
 *     [tokens][heads][head_dim] with a token stride and a head stride given in
 *     elements (both multiples of 8, head_dim contiguous).
 *   - Errors: argument, shape and capacity errors are returned before any work
 *     is enqueued and leave every state unchanged.  Errors found on the device
 *     (a bounded wait that ran out, an inconsistent mask buffer) are written to
 *     the cache's device error word and read by nomas_device_status.
 *   - Streams: nomas_stream is the CUDA runtime's cudaStream_t; NULL means the
 *     legacy default stream.  All work of one call goes to that stream.
 *   - Supported head_dim: 64 and 128.  Supported query rows: video tokens of
 *     the current segment.
 */
#ifndef NOMAS_H
#define NOMAS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nomas_stream;

typedef enum {
    NOMAS_OK = 0,
    NOMAS_EINVAL = -1,        /* bad argument, shape, stride or alignment */
    NOMAS_ECAPACITY = -2,     /* ring or head store would overflow */
    NOMAS_ECUDA = -3,         /* a CUDA runtime / driver call failed */
    NOMAS_ETIMEOUT = -4,      /* a bounded device wait ran out (device error word) */
    NOMAS_EDEVICE = -5,       /* inconsistent device data, e.g. a stale mask buffer */
    NOMAS_EUNSUPPORTED = -6,  /* head_dim or size not supported */
    NOMAS_ESTATE = -7,        /* call order or cache state does not allow the call */
    NOMAS_ERANGE = -8         /* an attention operand outside the supported range (device error word) */
} nomas_status;

/* Device buffers of a cache, all caller-owned; sizes from nomas_kv_cache_bytes.
 * Let C = capacity_frames, T = tokens_per_frame, H = heads, D = head_dim, S = head_store_tokens.
 *   K8, V8   int8  [H][C*T][D]   ring of latent-frame slots; frame g lives in slot g mod C
 *   KS, VS   fp32  [H][C*T]      one scale per (token, head): value = code * scale
 *   HK8, HV8 int8  [H][S][D]     description heads of appended segments, in append order
 *   HKS, HVS fp32  [H][S]
 *   ERR      int32 [4]           device error word (first error wins) + diagnostics
 */
enum {
    NOMAS_BUF_K8 = 0, NOMAS_BUF_V8, NOMAS_BUF_KS, NOMAS_BUF_VS,
    NOMAS_BUF_HK8, NOMAS_BUF_HV8, NOMAS_BUF_HKS, NOMAS_BUF_HVS,
    NOMAS_BUF_ERR, NOMAS_NBUF
};

typedef struct {
    int32_t heads;             /* H, >= 1 */
    int32_t head_dim;          /* D, 64 or 128 */
    int32_t tokens_per_frame;  /* T, tokens of one latent frame (880 at 1280x704) */
    int32_t window_frames;     /* W, retained history frames; 0 = keep full history */
    int32_t capacity_frames;   /* C, ring slots; >= W when W > 0 */
    int32_t head_store_tokens; /* S, capacity of the description-head store */
} nomas_cache_dims;

/* One action tail: `len` text tokens visible to query latent frames f0 <= t < f1
 * (segment-local frames) of its own segment only. */
typedef struct { int32_t len, f0, f1; } nomas_tail;

/* Text layout of the current segment: head_len description-head tokens followed
 * by the tails in order.  n_frames latent frames of T video tokens each. */
typedef struct {
    int32_t n_frames;
    int32_t head_len;
    int32_t n_tails;           /* <= NOMAS_MAX_TAILS */
    const nomas_tail *tails;   /* host pointer */
} nomas_segment_text;

#define NOMAS_MAX_TAILS 64

/* Host-mirrored ring state (deterministic from the append sequence). */
typedef struct {
    int64_t frames_appended;   /* global latent frames appended so far */
    int32_t retained_frames;   /* frames visible as history to the next segment */
    int32_t first_slot;        /* ring slot of the oldest retained frame */
    int64_t history_tokens;    /* retained_frames * T */
    int64_t head_tokens;       /* description-head tokens in the store */
    int32_t segments;          /* successful appends */
    int32_t _pad;
} nomas_cache_state;

typedef struct nomas_kv_cache nomas_kv_cache;

/* Total bytes of the cache's device buffers; out_sizes (nullable) receives each
 * buffer's size.  Returns 0 on invalid dims. */
size_t nomas_kv_cache_bytes(const nomas_cache_dims *dims, size_t out_sizes[NOMAS_NBUF]);

/* Create a host handle over caller-owned device buffers (bufs[i] sized by
 * nomas_kv_cache_bytes, 16-byte aligned).  Clears the device error word on
 * `stream`.  The cache starts empty. */
int nomas_kv_cache_init(nomas_kv_cache **out, const nomas_cache_dims *dims, void *const bufs[NOMAS_NBUF],
                        nomas_stream stream);

/* Free the host handle only; the device buffers stay the caller's. */
int nomas_kv_cache_destroy(nomas_kv_cache *cache);

int nomas_kv_cache_state(const nomas_kv_cache *cache, nomas_cache_state *out);

/* Quantise a finished segment's K/V and write them into the ring (fluxbbs.com
 * 单卡 4090 怎么做到的, first and second techniques; 架构 for the cache).
 *   k, v      bf16 [n_frames*T][H][D], strides tok_stride / head_stride (elements)
 *   head_k/v  bf16 [head_len][H][D], same strides; may be NULL when head_len == 0
 * Per (token, head): a = max|x|, s = a/127 (fp32, round to nearest), code =
 * clamp(rint(x/s), -127, 127) with fp32 division and round-half-even; a == 0
 * gives s = 0 and codes 0.  Frame f of the segment gets global index
 * g = frames_appended + f and ring slot g mod C; with a window W only frames
 * f >= n_frames - W are written (older ones would leave the window at once).
 * The description head is appended to the head store; action tails are never
 * cached.  Errors: NOMAS_ECAPACITY if the head store would overflow or, with
 * W == 0, the ring would; the cache is then unchanged. */
int nomas_kv_append(nomas_kv_cache *cache, const void *k, const void *v, int64_t tok_stride,
                    int64_t head_stride, int32_t n_frames, const void *head_k, const void *head_v,
                    int32_t head_len, nomas_stream stream);

/* ------------------------------------------------------------------------------------------------
 * Archive of evicted frames and selection of the retained history (hyphentech.top, config table:
 * in the single-GPU setting the GPU keeps at most 18 history latent frames and earlier history is
 * archived to CPU).  The pages say no more; this library's reading: a frame about to leave the window
 * can first be copied out as it stands (its INT8 codes and scales: a "record"), and the retained
 * history can be set to any list of at most min(W, NOMAS_MAX_SELECT_FRAMES) frames, each retained now
 * or given by its record, in the order listed -- which is then the history's age order for the mask,
 * the sparse selection and the attention.  Later appends add frames at the new end and drop from the
 * old end, the same window as before.  Without a selection nothing changes: frame g stays in ring
 * slot g mod C.
 * ------------------------------------------------------------------------------------------------ */
#define NOMAS_MAX_SELECT_FRAMES 64

/* Bytes of one frame record: K codes int8 [H][T][D], V codes int8 [H][T][D], K scales fp32 [H][T],
 * V scales fp32 [H][T], in that order (0 on invalid dims). */
size_t nomas_kv_frame_record_bytes(const nomas_cache_dims *dims);

/* The retained frames (global indices, age order) into frames[0 .. *n), at most max_frames of them
 * (NOMAS_ECAPACITY if more are retained). */
int nomas_kv_retained(const nomas_kv_cache *cache, int64_t *frames, int32_t max_frames, int32_t *n);

/* The retained frames (oldest first) that an append of n_frames would drop from the window, into
 * frames[0 .. *n) (none without a window). */
int nomas_kv_evicted_by(const nomas_kv_cache *cache, int32_t n_frames, int64_t *frames, int32_t max_frames,
                        int32_t *n);

/* Copy retained frame `frame` out of the cache into `record` (host memory of
 * nomas_kv_frame_record_bytes bytes; pinned memory makes the copies asynchronous).  The record is
 * complete once `stream` has reached this point.  Errors: NOMAS_EINVAL if the frame is not retained. */
int nomas_kv_archive(const nomas_kv_cache *cache, int64_t frame, void *record, nomas_stream stream);

/* Make frames[0 .. n) the retained history, in that age order.  A frame retained now keeps its data;
 * any other frame is copied in from records[i] (a host record written by nomas_kv_archive; records[i]
 * may be NULL for retained frames, and `records` may be NULL when every frame is retained).  Needs a
 * window (W > 0) with W <= NOMAS_MAX_SELECT_FRAMES and n <= W, no repeated frame: NOMAS_EUNSUPPORTED /
 * NOMAS_EINVAL before anything is enqueued.  Incoming frames go to slots no kept frame uses; if a copy
 * fails (NOMAS_ECUDA) the retained history is undefined.  Records are read on `stream` (keep them alive
 * and unchanged until it has passed this point). */
int nomas_kv_select(nomas_kv_cache *cache, const int64_t *frames, int32_t n, const void *const *records,
                    nomas_stream stream);

#define NOMAS_MODE_DENSE 0
#define NOMAS_MODE_SPARSE 1
/* Text query rows of the current segment (the text stream of the double-stream joint attention,
 * papers.ananclaw.com "干货攻略", 这是什么), always dense.  The pages say who may see the text, not what
 * the text sees; this library's reading: a description-head row sees the retained history, earlier
 * heads, all current video and the current head, but no action tail (the head is cached and visible
 * across segments, so it must not carry the segment's actions); a row of tail a (window [f0, f1))
 * sees the history, earlier heads and the current head, the current video frames t with
 * f0 <= t < f1, and the tails whose window shares a frame with a's (itself included).  In this mode
 * nomas_mask_build needs no q / kcur, and nomas_attn_run / nomas_attn_fwd read q as the text queries
 * [text_tokens][H][D] and write out [text_tokens][H][D] and lse [H][text_tokens].  A row with no
 * visible key (possible only in degenerate layouts) gets output 0. */
#define NOMAS_MODE_TEXT 2

/* Where mask_build puts its results inside the caller's mask buffer.
 * Key order for tiles and classes: retained history (age order), description
 * heads of earlier segments, current video, current text (head then tails);
 * every region is cut into 128-key tiles from its first key.  Query blocks are
 * 128 current-video rows. */
typedef struct {
    int32_t mode, head_dim, heads, n_qblocks;
    int32_t n_tiles;           /* KV tiles over all four regions */
    int32_t n_hist_tiles, n_head_tiles, n_cur_tiles, n_text_tiles;
    int32_t n_cand;            /* sparse candidates: history tiles then current tiles */
    int32_t keep;              /* kept candidates per (head, query block); 0 in dense mode */
    int32_t n_lists, list_cap; /* per-CTA tile lists used by nomas_attn_fwd */
    int32_t _pad;
    int64_t history_tokens, head_tokens, n_query, text_tokens;
    size_t off_class;          /* int8  [n_qblocks][n_tiles]: 0 SKIP, 1 FULL, 2 PARTIAL */
    size_t off_sel;            /* int32 [H][n_qblocks][keep]: kept candidates, score desc then index asc */
    size_t off_score;          /* fp32  [H][n_qblocks][n_cand] */
    size_t off_qmean;          /* fp32  [H][n_qblocks][D]   (scratch) */
    size_t off_kmean;          /* fp32  [H][n_cand][D]      (scratch) */
    size_t off_txtwin;         /* int32 [text_tokens][2]: visible frame window [lo, hi) per text key */
    size_t off_count;          /* int32 [n_lists] */
    size_t off_list;           /* int32x4 [n_lists][list_cap] */
    size_t total_bytes;
} nomas_mask_layout;

/* Fill `out` for the current cache state and segment text.  keep_frac in (0, 1]
 * (sparse only): keep = clamp(ceil(n_cand * keep_frac), 1, n_cand), ceil taken in
 * double precision of the float value.  Sparse mode supports at most
 * NOMAS_MAX_SPARSE_CANDIDATES candidate blocks (about a million history plus current tokens);
 * more return NOMAS_EUNSUPPORTED. */
#define NOMAS_MAX_SPARSE_CANDIDATES 8192
int nomas_mask_layout_query(const nomas_kv_cache *cache, const nomas_segment_text *seg, int mode,
                            float keep_frac, nomas_mask_layout *out);

/* Bytes of the mask buffer (0 on invalid arguments). */
size_t nomas_mask_bytes(const nomas_kv_cache *cache, const nomas_segment_text *seg, int mode, float keep_frac);

/* Build the visibility classes and per-CTA tile lists (fluxbbs.com 架构) and,
 * in sparse mode, the kept candidate blocks (same page, fourth technique of
 * 单卡 4090 怎么做到的; the ranking rule is this library's own: per head and
 * query block, score = fmaf chain over channels of the fp32 mean of the block's
 * queries and the fp32 mean of the candidate's keys, history keys taken as
 * float(code) * scale, sums in ascending token order, mean = sum / n_valid; ranked by
 * score descending then candidate index ascending, with a NaN score ranked as -inf).
 *   q, kcur   bf16 [n_frames*T][H][D] (sparse mode only; NULL allowed in dense)
 *   mask_buf  device buffer of nomas_mask_bytes bytes, 16-byte aligned
 * The result is valid for this cache state; an append in between makes
 * nomas_attn_fwd report NOMAS_EDEVICE through the error word. */
int nomas_mask_build(const nomas_kv_cache *cache, const nomas_segment_text *seg, int mode, float keep_frac,
                     const void *q, const void *kcur, int64_t tok_stride, int64_t head_stride, void *mask_buf,
                     nomas_stream stream);

/* Allocation-free variant of nomas_mask_build (the pages have no counterpart: this is an interface
 * convenience of this library).  Some callers cannot allocate device memory on the path that builds
 * the mask: a host framework that owns the whole device pool and hands plugins no allocator, or a
 * latency-critical serving loop in which a cudaMalloc could synchronise the device.  In sparse mode
 * nomas_mask_build keeps the pooled per-block query and key means (scratch) inside the caller's
 * mask buffer; this variant keeps them in a file-scope device array of NOMAS_STATIC_POOL_FLOATS
 * floats (8 MiB) that every GPU which loads the library holds until the process exits.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   Arguments, mask buffer layout and results: as nomas_mask_build (dense mode forwards to it
 *   unchanged, it needs no scratch).  The qmean / kmean regions of mask_buf are left untouched.
 *   Limit: heads * (n_qblocks + n_cand) * head_dim <= NOMAS_STATIC_POOL_FLOATS, else
 *   NOMAS_ECAPACITY before anything is enqueued (1280x704 shape with an 18-frame history:
 *   1.10 M floats; 480x832: 0.22 M).
 *   The first call on a device looks up the array's device address (once per device, with that
 *   device current); make that first call before any stream capture.
 *   All calls on a device share the one array and it keeps the last call's contents; every element
 *   a call reads it has written first, so nothing needs clearing.  Calls that overlap on the GPU
 *   (different streams, no ordering between them) race on the array. */
#define NOMAS_STATIC_POOL_FLOATS ((size_t)2 << 20)
int nomas_mask_build_static(const nomas_kv_cache *cache, const nomas_segment_text *seg, int mode,
                            float keep_frac, const void *q, const void *kcur, int64_t tok_stride,
                            int64_t head_stride, void *mask_buf, nomas_stream stream);

/* Bytes of the workspace nomas_attn_fwd needs for this cache and segment text (0 on invalid
 * arguments).  The size depends only on the cache dimensions and the segment text, not on how much
 * history is retained.  nomas_attn_fwd fills it with its operand copies: fp16 keys [H][n][D] and
 * transposed fp16 values [H][D][n] of the current segment and the text, and the INT8 codes of the
 * retained history (in age order, with its scales) and of the description heads widened to exact
 * fp16 integers in the same two layouts (no scale applied).  1280x704 shape with an 18-frame
 * history: 0.36 GB. */
size_t nomas_attn_workspace_bytes(const nomas_kv_cache *cache, const nomas_segment_text *seg);

/* Masked (or block-sparse) attention of the current segment's video queries over the retained INT8
 * history, earlier description heads (INT8), the current segment's video and its text, with the
 * visibility of nomas_mask_build (fluxbbs.com 架构; sparse mode: same page, 单卡 4090 怎么做到的).
 * Per head h and query row i:
 *     O[i,h] = sum_j softmax_j(softmax_scale * q_i . k^_j) v^_j   over visible j
 * with k^ = code * scale and v^ = code * scale for cached keys and values.  The codes enter the
 * tensor core exactly: the key scale multiplies the fp32 score and the value scale the fp32
 * probability, which is then rounded once to fp16 (so each term p * v^ is fp16(p * scale) * code).
 * The QK^T and PV products run on the tensor cores with fp16 operands and fp32 accumulation; bf16
 * inputs convert to fp16 exactly for magnitudes in [2^-14, 65504] (smaller magnitudes keep fp16's
 * 2^-24 absolute resolution).
 * Supported range, checked on the device: every q, kcur, vcur, ktxt, vtxt element finite with
 * magnitude below 65520 (it must not round to an fp16 infinity), and every cached value scale at
 * most 65504 / 64 = 1023.5 (a (token, head) absmax of about 1.3e5 at append time) with finite key
 * scales.  A violation records NOMAS_ERANGE in the device error word (read by
 * nomas_device_status); the call still completes and the outputs of the affected rows are
 * undefined.
 *   q, kcur, vcur  bf16 [n_frames*T][H][D];  ktxt, vtxt bf16 [text_tokens][H][D]
 *                  (NULL allowed when the segment has no text); all share tok_stride / head_stride
 *   out            fp32 [n_frames*T][H][D], contiguous
 *   lse            fp32 [H][n_frames*T] natural-log sum of exp of the scaled scores, nullable
 *   workspace      device buffer of nomas_attn_workspace_bytes bytes, 16-byte aligned, caller-owned;
 *                  overwritten by the call (calls that share it must not overlap on the GPU) */
int nomas_attn_fwd(const nomas_kv_cache *cache, const nomas_segment_text *seg, int mode, float keep_frac,
                   const void *mask_buf, const void *q, const void *kcur, const void *vcur, const void *ktxt,
                   const void *vtxt, int64_t tok_stride, int64_t head_stride, float softmax_scale, float *out,
                   float *lse, void *workspace, nomas_stream stream);

/* The two halves of nomas_attn_fwd, for callers that time or schedule them separately
 * (nomas_attn_fwd enqueues exactly nomas_attn_prepare followed by nomas_attn_run).
 *
 * nomas_attn_prepare: the HBM-bound pre-pass.  Writes into `workspace` the fp16 copies of kcur, vcur,
 * ktxt, vtxt (keys [H][n][D], values transposed [H][D][n]) and the retained history's and description
 * heads' INT8 codes widened to exact fp16 (with the history's scales in age order), plus a header that
 * records the cache state and segment it was prepared for.  Arguments as nomas_attn_fwd.
 *
 * nomas_attn_run: the masked (or block-sparse) attention kernel over a prepared workspace; q is read
 * here.  The kernel checks the workspace header (and the mask buffer's) against the cache state and
 * segment of the call: a workspace prepared before a later append, for another segment, or never
 * prepared records NOMAS_EDEVICE in the device error word and leaves `out` unwritten.  The workspace
 * holds the K/V values of the last prepare: a caller that changes kcur / vcur / ktxt / vtxt must
 * prepare again. */
int nomas_attn_prepare(const nomas_kv_cache *cache, const nomas_segment_text *seg, const void *kcur,
                       const void *vcur, const void *ktxt, const void *vtxt, int64_t tok_stride,
                       int64_t head_stride, void *workspace, nomas_stream stream);
int nomas_attn_run(const nomas_kv_cache *cache, const nomas_segment_text *seg, int mode, float keep_frac,
                   const void *mask_buf, const void *q, int64_t tok_stride, int64_t head_stride,
                   float softmax_scale, float *out, float *lse, void *workspace, nomas_stream stream);

/* Diagnostic: retained history in age order, dequantised as fp32 code * scale.
 *   k_out, v_out  fp32 [history_tokens][H][D] */
int nomas_kv_dequant(const nomas_kv_cache *cache, float *k_out, float *v_out, nomas_stream stream);

/* ------------------------------------------------------------------------------------------
 * INT8-weight / BF16-compute linear layer of the DiT (fluxbbs.com "单卡 4090 怎么做到的", first
 * technique: model weights are stored as INT8 with float scale factors and dequantised back to BF16
 * at compute time; the DiT's linear layers compute in BF16).  The pages give no formula; reading:
 *   - one scale per output channel: row n of W [N][K] is quantised as one vector with the K/V
 *     quantiser above (s_n = RN(absmax / 127), codes rint(w / s_n) half-even);
 *   - dequantised weight w_nk = bf16(RN(fp32(q_nk * s_n)));
 *   - y = x W^T with bf16 x, fp32 accumulation.
 * Layouts: x bf16 [M][K] row pitch ldx elements, W (bf16 or codes) [N][K] row pitch ldw (codes: K),
 * y [M][N] row pitch ldy >= N elements, fp32 (NOMAS_DTYPE_F32) or bf16 (NOMAS_DTYPE_BF16).  Every
 * pointer is device memory, caller-owned, 16-byte aligned; K, ldx and ldw are multiples of 8.
 * `status` is a caller-owned device int32[4] error word (same format as a cache's): a bounded wait
 * that runs out records NOMAS_ETIMEOUT there; read and clear it with nomas_status_read.
 * Errors (returned before anything is enqueued): NOMAS_EINVAL for a null or misaligned pointer,
 * a size below 1 or a pitch that breaks the rules above; NOMAS_ECUDA for a failed launch. */
#define NOMAS_DTYPE_F32 0
#define NOMAS_DTYPE_BF16 1

/* Quantise bf16 weights w [N][K] (row pitch ldw) into codes int8 [N][K] and scales fp32 [N]. */
int nomas_w8_quantize(const void *w, int64_t n_out, int64_t k_in, int64_t ldw, int8_t *codes, float *scales,
                      nomas_stream stream);
/* Dequantise codes int8 [N][K] with scales fp32 [N] into bf16 weights w [N][K] (dense). */
int nomas_w8_dequant(const int8_t *codes, const float *scales, int64_t n_out, int64_t k_in, void *w,
                     nomas_stream stream);
/* y = x W^T for bf16 x [M][K] and bf16 W [N][K]: tcgen05 tiles of 128 x 256, fp32 accumulation in TMEM. */
int nomas_linear_bf16(const void *x, int64_t m, int64_t k_in, int64_t ldx, const void *w, int64_t n_out,
                      int64_t ldw, void *y, int64_t ldy, int y_dtype, int32_t *status, nomas_stream stream);
/* Bytes of the transient bf16 weights nomas_w8a16_linear dequantises into: N * K * 2. */
size_t nomas_w8a16_workspace_bytes(int64_t n_out, int64_t k_in);
/* nomas_w8_dequant into `workspace`, then nomas_linear_bf16 with those weights. */
int nomas_w8a16_linear(const void *x, int64_t m, int64_t k_in, int64_t ldx, const int8_t *codes,
                       const float *scales, int64_t n_out, void *y, int64_t ldy, int y_dtype, void *workspace,
                       int32_t *status, nomas_stream stream);
/* Synchronise `stream`, read and clear a linear layer's device error word. */
int nomas_status_read(int32_t *status, nomas_stream stream);

/* Synchronise `stream`, read and clear the device error word.  Returns NOMAS_OK
 * or the first device-side error recorded since the last call. */
int nomas_device_status(const nomas_kv_cache *cache, nomas_stream stream);

const char *nomas_status_string(int status);

/* Diagnostic text of the last NOMAS_ECUDA returned on the calling thread: the CUDA call that
 * failed and its error string ("" if none).  Valid until the next failing call on this thread. */
const char *nomas_last_error(void);

/* Test and diagnostic hook: the limit, in nanoseconds, of every bounded wait inside the attention
 * and append kernels, the sparse selection's pooling kernel and the linear layer (process-wide, default
 * 2 000 000 000 = 2 s; it applies to later calls).  A
 * wait that runs out records NOMAS_ETIMEOUT in the cache's device error word, and every role of the
 * CTA then leaves its loop, lets its in-flight copies and MMAs complete and releases TMEM, so the
 * device stays usable; the call's output is then undefined.  A limit of 0 makes a wait that its
 * first poll does not satisfy give up at once, which exercises that path.  Returns the previous
 * limit. */
uint64_t nomas_set_wait_limit_ns(uint64_t limit_ns);

/* Tuning and test hook: the number of shares a NOMAS_MODE_TEXT call cuts each key list into.  The
 * text query rows fill only ceil(text_tokens / 128) x heads CTAs and their lists differ in length, so
 * each list is cut into shares of ceil(list capacity / shares) entries, one CTA each; a CTA writes its
 * output without normalisation plus (running maximum, row sum) per row to the workspace, and a merge
 * kernel forms out and lse from the shares (the softmax merge of disjoint key sets, exact up to
 * rounding order).  By default (shares = 0) the call picks the count from the CTA count, the SM
 * count and the list capacity; 1 to 16 forces that count (1: one CTA per list, no merge); other
 * values select the default.  Process-wide, applies to later calls; returns the previous setting. */
int nomas_set_text_split(int shares);

/* Tuning and test hook: which attention kernel nomas_attn_run uses at head_dim 128.  0 (default): one
 * CTA per pair of 128-row query blocks that share a tile list for NOMAS_MODE_DENSE when the pairs fill
 * the SMs in fewer waves of work (the two blocks' softmax warps alternate on the tensor pipe, and each
 * K / V^T tile is staged once for both), else and for the sparse and text-row modes (whose two blocks
 * share fewer tiles) one CTA per query block; 1: one CTA per
 * query block in every mode (the kernel head_dim 64 always uses); 2: block pairs in every mode.  All
 * compute the same function (same operand precision and softmax arithmetic; results agree up to the
 * order of the fp32 row-sum additions).  Other values select 0.  Process-wide, applies to later
 * calls; returns the previous setting. */
int nomas_set_attn_kernel(int which);

#ifdef __cplusplus
}
#endif
#endif /* NOMAS_H */
