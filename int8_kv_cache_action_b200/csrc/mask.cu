// nomas_mask_build: visibility classes per (128-query block, 128-key tile), per-CTA tile lists for
// nomas_attn_fwd and, in sparse mode, the kept candidate video blocks.
//
// Visibility (fluxbbs.com "架构"): every video query of the current segment sees the retained
// history, the description heads of earlier segments, all current-segment video (bidirectional) and
// the current description head; action tail a is visible to query frame t iff f0_a <= t < f1_a.
// Sparse mode (same page, fourth technique of "单卡 4090 怎么做到的"): keep ceil(keep_frac * n)
// candidate video blocks per head and query block, ranked by a fixed-order fp32 score (this
// library's own rule; see nomas.h).  All integer work is exact; the fp32 steps use explicit
// round-to-nearest intrinsics so the result does not depend on contraction or operation order.
#include <cmath>

#include "common.cuh"

namespace nomas {

struct MaskParams {
    MaskHeader hdr;
    int32_t n_tails;
    int32_t head_len;
    nomas_tail tails[NOMAS_MAX_TAILS];
    int32_t T, H, D;
    int64_t Lh, Lp, Nq, Lt;
    int32_t n_qb, n_tiles, n_hist_tiles, n_head_tiles, n_cur_tiles, n_text_tiles, n_cand, keep, n_lists, list_cap;
    uint8_t *buf;
    nomas_mask_layout lay;
    // sparse inputs
    const __nv_bfloat16 *q, *kcur;
    int64_t tok_stride, head_stride;
    const int8_t *k8;
    const float *ks;
    int64_t ring_tokens, first_tok;
};

struct TileInfo {
    int kind;
    int64_t start;
    int32_t count;
};

__device__ __forceinline__ TileInfo tile_info(const MaskParams &p, int j) {
    TileInfo t;
    int64_t len;
    if (j < p.n_hist_tiles) {
        t.kind = kKindHist;
        len = p.Lh;
    } else if ((j -= p.n_hist_tiles) < p.n_head_tiles) {
        t.kind = kKindPriorHead;
        len = p.Lp;
    } else if ((j -= p.n_head_tiles) < p.n_cur_tiles) {
        t.kind = kKindCur;
        len = p.Nq;
    } else {
        j -= p.n_cur_tiles;
        t.kind = kKindText;
        len = p.Lt;
    }
    t.start = (int64_t)j * kTile;
    const int64_t rem = len - t.start;
    t.count = (int32_t)(rem < kTile ? rem : kTile);
    return t;
}

// Header + per-text-token visibility window [lo, hi) in segment-local latent frames.
__global__ void mask_prep_kernel(MaskParams p) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) *reinterpret_cast<MaskHeader *>(p.buf) = p.hdr;
    if (i >= p.Lt) return;
    int2 w = make_int2(0, kAlwaysHi);
    if (i >= p.head_len) {
        int64_t at = p.head_len;
        for (int a = 0; a < p.n_tails; ++a) {
            const int64_t end = at + p.tails[a].len;
            if (i < end) {
                w = make_int2(p.tails[a].f0, p.tails[a].f1);
                break;
            }
            at = end;
        }
    }
    reinterpret_cast<int2 *>(p.buf + p.lay.off_txtwin)[i] = w;
}

// One thread per (query block, KV tile): SKIP / FULL / PARTIAL over valid rows and valid keys.
__global__ void class_map_kernel(MaskParams p) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.n_qb * p.n_tiles) return;
    const int b = (int)(idx / p.n_tiles);
    const int j = (int)(idx % p.n_tiles);
    const TileInfo ti = tile_info(p, j);
    int8_t cls = 1;  // FULL
    if (ti.kind == kKindText) {
        const int2 *win = reinterpret_cast<const int2 *>(p.buf + p.lay.off_txtwin);
        const int64_t r0 = (int64_t)b * kTile;
        const int64_t r1 = (r0 + kTile < p.Nq) ? r0 + kTile : p.Nq;
        int64_t vis = 0;
        const int64_t total = (r1 - r0) * ti.count;
        for (int64_t t = r0 / p.T; t <= (r1 - 1) / p.T; ++t) {
            const int64_t a0 = t * p.T > r0 ? t * p.T : r0;
            const int64_t a1 = (t + 1) * p.T < r1 ? (t + 1) * p.T : r1;
            int64_t nk = 0;
            for (int k = 0; k < ti.count; ++k) {
                const int2 w = win[ti.start + k];
                nk += (w.x <= t && t < w.y) ? 1 : 0;
            }
            vis += (a1 - a0) * nk;
        }
        cls = vis == total ? 1 : (vis == 0 ? 0 : 2);
    }
    reinterpret_cast<int8_t *>(p.buf + p.lay.off_class)[idx] = cls;
}

__device__ __forceinline__ int mask_flag(int8_t cls, int32_t count) { return (cls == 2 || count < kTile); }

// Dense lists: one thread per pair of query blocks (one attention CTA); lists are head-independent.
__global__ void lists_dense_kernel(MaskParams p) {
    // one warp per list: lanes test 32 tiles at a time, kept tiles are compacted in index order
    const int pr = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (pr >= p.n_lists) return;   // warp-uniform
    const int b0 = 2 * pr, b1 = 2 * pr + 1;
    const int8_t *cls = reinterpret_cast<const int8_t *>(p.buf + p.lay.off_class);
    int4 *out = reinterpret_cast<int4 *>(p.buf + p.lay.off_list) + (int64_t)pr * p.list_cap;
    int n = 0;
    for (int j0 = 0; j0 < p.n_tiles; j0 += 32) {
        const int j = j0 + lane;
        int8_t c0 = 0, c1 = 0;
        if (j < p.n_tiles) {
            c0 = cls[(int64_t)b0 * p.n_tiles + j];
            c1 = b1 < p.n_qb ? cls[(int64_t)b1 * p.n_tiles + j] : 0;
        }
        const bool keep = c0 != 0 || c1 != 0;
        const uint32_t m = __ballot_sync(0xffffffffu, keep);
        if (keep) {
            const TileInfo ti = tile_info(p, j);
            int f = ti.kind;
            if (c0) f |= kUse0 | (mask_flag(c0, ti.count) ? kMask0 : 0);
            if (c1) f |= kUse1 | (mask_flag(c1, ti.count) ? kMask1 : 0);
            out[n + __popc(m & ((1u << lane) - 1u))] = make_int4(f, (int)ti.start, ti.count, j);
        }
        n += __popc(m);
    }
    if (lane == 0) reinterpret_cast<int32_t *>(p.buf + p.lay.off_count)[pr] = n;
}

// ------------------------------------------------------------------------------------------------
// sparse selection (fixed-order fp32)
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_at(const __nv_bfloat16 *x, int64_t i) { return __bfloat162float(x[i]); }

// qmean[h][b][c]: sequential fp32 sum over the block's valid rows in ascending order, one division.
__global__ void qmean_kernel(MaskParams p) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n = (int64_t)p.H * p.n_qb * p.D;
    if (idx >= n) return;
    const int c = (int)(idx % p.D);
    const int64_t hb = idx / p.D;
    const int b = (int)(hb % p.n_qb);
    const int h = (int)(hb / p.n_qb);
    const int64_t r0 = (int64_t)b * kTile;
    const int nv = (int)((r0 + kTile < p.Nq) ? kTile : p.Nq - r0);
    float acc = 0.0f;
    for (int i = 0; i < nv; ++i)
        acc = __fadd_rn(acc, bf16_at(p.q, (r0 + i) * p.tok_stride + (int64_t)h * p.head_stride + c));
    reinterpret_cast<float *>(p.buf + p.lay.off_qmean)[idx] = __fdiv_rn(acc, (float)nv);
}

// kmean[h][cand][c]: history candidates dequantise with one fp32 multiply (code * scale); sums in
// ascending token order from +0, one division.  The ring row advances incrementally (no modulo per
// token).
__device__ __forceinline__ float kmean_value(const MaskParams &p, int64_t idx) {
    const int c = (int)(idx % p.D);
    const int64_t hc = idx / p.D;
    const int cand = (int)(hc % p.n_cand);
    const int h = (int)(hc / p.n_cand);
    float acc = 0.0f;
    int nv;
    if (cand < p.n_hist_tiles) {
        const int64_t a0 = (int64_t)cand * kTile;
        nv = (int)((a0 + kTile < p.Lh) ? kTile : p.Lh - a0);
        int64_t phys = (p.first_tok + a0) % p.ring_tokens;
        const int64_t base = (int64_t)h * p.ring_tokens;
        for (int i = 0; i < nv; ++i) {
            const int64_t r = base + phys;
            acc = __fadd_rn(acc, __fmul_rn((float)p.k8[r * p.D + c], p.ks[r]));
            if (++phys == p.ring_tokens) phys = 0;
        }
    } else {
        const int64_t a0 = (int64_t)(cand - p.n_hist_tiles) * kTile;
        nv = (int)((a0 + kTile < p.Nq) ? kTile : p.Nq - a0);
        for (int i = 0; i < nv; ++i)
            acc = __fadd_rn(acc, bf16_at(p.kcur, (a0 + i) * p.tok_stride + (int64_t)h * p.head_stride + c));
    }
    return __fdiv_rn(acc, (float)nv);
}

__global__ void kmean_kernel(MaskParams p) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.H * p.n_cand * p.D) return;
    reinterpret_cast<float *>(p.buf + p.lay.off_kmean)[idx] = kmean_value(p, idx);
}

// score[h][b][cand] = fmaf chain over channels in ascending order from +0.0f.  One block covers
// kScoreQB query blocks of one head; candidate means are staged 32 at a time in shared memory (rows
// padded by one float so the 32 lanes of a warp, one candidate each, hit distinct banks), and each
// thread runs the chain of one (query block, candidate) pair.
constexpr int kScoreQB = 8;

__device__ __forceinline__ void score_block(const MaskParams &p, const float *qmean_all, const float *kmean_all) {
    extern __shared__ float sh[];
    const int D = p.D;
    const int qb_chunks = (p.n_qb + kScoreQB - 1) / kScoreQB;
    const int h = blockIdx.x / qb_chunks;
    const int b0 = (blockIdx.x % qb_chunks) * kScoreQB;
    float *qm_s = sh;                     // [kScoreQB][D]
    float *km_s = sh + kScoreQB * D;      // [32][D + 1]
    for (int i = threadIdx.x; i < kScoreQB * D; i += blockDim.x) {
        const int b = b0 + i / D;
        qm_s[i] = b < p.n_qb ? qmean_all[((int64_t)h * p.n_qb + b) * D + i % D] : 0.0f;
    }
    const int bl = threadIdx.x >> 5, cl = threadIdx.x & 31;
    const int b = b0 + bl;
    const float *km = kmean_all + (int64_t)h * p.n_cand * D;
    float *sc = reinterpret_cast<float *>(p.buf + p.lay.off_score);
    for (int c0 = 0; c0 < p.n_cand; c0 += 32) {
        __syncthreads();
        for (int i = threadIdx.x; i < 32 * D; i += blockDim.x) {
            const int cand = c0 + i / D;
            km_s[(i / D) * (D + 1) + i % D] = cand < p.n_cand ? km[(int64_t)cand * D + i % D] : 0.0f;
        }
        __syncthreads();
        const int cand = c0 + cl;
        if (b < p.n_qb && cand < p.n_cand) {
            const float *q = qm_s + bl * D, *k = km_s + cl * (D + 1);
            float acc = 0.0f;
            for (int c = 0; c < D; ++c) acc = __fmaf_rn(q[c], k[c], acc);
            sc[((int64_t)h * p.n_qb + b) * p.n_cand + cand] = acc;
        }
    }
}

__global__ void __launch_bounds__(32 * kScoreQB) score_kernel(MaskParams p) {
    score_block(p, reinterpret_cast<const float *>(p.buf + p.lay.off_qmean),
                reinterpret_cast<const float *>(p.buf + p.lay.off_kmean));
}

static size_t score_smem(int D) { return (size_t)(kScoreQB * D + 32 * (D + 1)) * sizeof(float); }
static unsigned score_grid(const MaskParams &p) { return (unsigned)(p.H * ((p.n_qb + kScoreQB - 1) / kScoreQB)); }

// Rank every candidate (score descending, index ascending); ranks below keep are written in order.
__global__ void select_kernel(MaskParams p) {
    extern __shared__ float sc_s[];
    const int hb = blockIdx.x;
    const float *sc = reinterpret_cast<const float *>(p.buf + p.lay.off_score) + (int64_t)hb * p.n_cand;
    for (int i = threadIdx.x; i < p.n_cand; i += blockDim.x) sc_s[i] = sc[i];
    __syncthreads();
    int32_t *sel = reinterpret_cast<int32_t *>(p.buf + p.lay.off_sel) + (int64_t)hb * p.keep;
    for (int i = threadIdx.x; i < p.n_cand; i += blockDim.x) {
        const float si = sc_s[i];
        int rank = 0;
        for (int j = 0; j < p.n_cand; ++j) {
            const float sj = sc_s[j];
            rank += (sj > si || (sj == si && j < i)) ? 1 : 0;
        }
        if (rank < p.keep) sel[rank] = i;
    }
}

// Sparse lists: one block per (head, pair); kept candidates in index order, then description
// heads of earlier segments (always visible), then text tiles by their dense class.
__global__ void lists_sparse_kernel(MaskParams p) {
    extern __shared__ uint32_t bits[];  // [2][words]
    const int n_pairs = (p.n_qb + 1) / 2;
    const int hp = blockIdx.x;           // h * n_pairs + pair
    const int h = hp / n_pairs, pr = hp % n_pairs;
    const int words = (p.n_cand + 31) / 32;
    for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) bits[i] = 0;
    __syncthreads();
    const int b0 = 2 * pr, b1 = 2 * pr + 1;
    const int32_t *sel = reinterpret_cast<const int32_t *>(p.buf + p.lay.off_sel);
    for (int q = 0; q < 2; ++q) {
        const int b = q ? b1 : b0;
        if (b >= p.n_qb) continue;
        const int32_t *s = sel + ((int64_t)h * p.n_qb + b) * p.keep;
        for (int i = threadIdx.x; i < p.keep; i += blockDim.x) {
            const int c = s[i];
            atomicOr(&bits[q * words + c / 32], 1u << (c % 32));
        }
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    const int8_t *cls = reinterpret_cast<const int8_t *>(p.buf + p.lay.off_class);
    int4 *out = reinterpret_cast<int4 *>(p.buf + p.lay.off_list) + (int64_t)hp * p.list_cap;
    int n = 0;
    const bool has1 = b1 < p.n_qb;
    for (int j = 0; j < p.n_tiles; ++j) {
        const TileInfo ti = tile_info(p, j);
        bool u0, u1;
        bool m0, m1;
        if (ti.kind == kKindHist || ti.kind == kKindCur) {
            const int cand = ti.kind == kKindHist ? j : j - p.n_head_tiles;
            u0 = (bits[cand / 32] >> (cand % 32)) & 1u;
            u1 = has1 && ((bits[words + cand / 32] >> (cand % 32)) & 1u);
            m0 = m1 = ti.count < kTile;
        } else {
            const int8_t c0 = cls[(int64_t)b0 * p.n_tiles + j];
            const int8_t c1 = has1 ? cls[(int64_t)b1 * p.n_tiles + j] : 0;
            u0 = c0 != 0;
            u1 = c1 != 0;
            m0 = mask_flag(c0, ti.count);
            m1 = mask_flag(c1, ti.count);
        }
        if (!u0 && !u1) continue;
        int f = ti.kind;
        if (u0) f |= kUse0 | (m0 ? kMask0 : 0);
        if (u1) f |= kUse1 | (m1 ? kMask1 : 0);
        out[n++] = make_int4(f, (int)ti.start, ti.count, j);
    }
    reinterpret_cast<int32_t *>(p.buf + p.lay.off_count)[hp] = n;
}

static unsigned nblk(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace nomas

using namespace nomas;

extern "C" int nomas_mask_build(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                                const void *q, const void *kcur, int64_t tok_stride, int64_t head_stride,
                                void *mask_buf, nomas_stream stream) {
    nomas_mask_layout lay;
    int rc = compute_mask_layout(c, seg, mode, keep_frac, &lay);
    if (rc) return rc;
    if (!mask_buf || !aligned16(mask_buf)) return NOMAS_EINVAL;
    const bool sp = mode == NOMAS_MODE_SPARSE;
    if (sp) {
        if (!q || !kcur || !aligned16(q) || !aligned16(kcur)) return NOMAS_EINVAL;
        if (tok_stride <= 0 || head_stride <= 0 || tok_stride % 8 || head_stride % 8) return NOMAS_EINVAL;
        if (lay.n_cand < 1) return NOMAS_EINVAL;
    }
    if (bind_device(c)) return NOMAS_ECUDA;
    MaskParams p{};
    const HistView hv = hist_view(c);
    p.hdr.magic = kMaskMagic;
    p.hdr.mode = mode;
    p.hdr.n_qblocks = lay.n_qblocks;
    p.hdr.n_lists = lay.n_lists;
    p.hdr.history_tokens = lay.history_tokens;
    p.hdr.head_tokens = lay.head_tokens;
    p.hdr.frames_appended = c->frames_appended;
    p.hdr.n_query = lay.n_query;
    p.hdr.text_tokens = lay.text_tokens;
    p.hdr.list_cap = lay.list_cap;
    p.hdr.keep = lay.keep;
    p.n_tails = seg->n_tails;
    p.head_len = seg->head_len;
    for (int i = 0; i < seg->n_tails; ++i) p.tails[i] = seg->tails[i];
    p.T = c->d.tokens_per_frame;
    p.H = c->d.heads;
    p.D = c->d.head_dim;
    p.Lh = lay.history_tokens;
    p.Lp = lay.head_tokens;
    p.Nq = lay.n_query;
    p.Lt = lay.text_tokens;
    p.n_qb = lay.n_qblocks;
    p.n_tiles = lay.n_tiles;
    p.n_hist_tiles = lay.n_hist_tiles;
    p.n_head_tiles = lay.n_head_tiles;
    p.n_cur_tiles = lay.n_cur_tiles;
    p.n_text_tiles = lay.n_text_tiles;
    p.n_cand = lay.n_cand;
    p.keep = lay.keep;
    p.n_lists = lay.n_lists;
    p.list_cap = lay.list_cap;
    p.buf = static_cast<uint8_t *>(mask_buf);
    p.lay = lay;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.kcur = static_cast<const __nv_bfloat16 *>(kcur);
    p.tok_stride = tok_stride;
    p.head_stride = head_stride;
    p.k8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_K8]);
    p.ks = static_cast<const float *>(c->buf[NOMAS_BUF_KS]);
    p.ring_tokens = hv.ring_tokens;
    p.first_tok = hv.first_tok;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    mask_prep_kernel<<<nblk(lay.text_tokens > 0 ? lay.text_tokens : 1, 256), 256, 0, st>>>(p);
    class_map_kernel<<<nblk((int64_t)lay.n_qblocks * lay.n_tiles, 256), 256, 0, st>>>(p);
    if (!sp) {
        lists_dense_kernel<<<nblk((int64_t)lay.n_lists * 32, 128), 128, 0, st>>>(p);
    } else {
        qmean_kernel<<<nblk((int64_t)p.H * p.n_qb * p.D, 256), 256, 0, st>>>(p);
        kmean_kernel<<<nblk((int64_t)p.H * p.n_cand * p.D, 256), 256, 0, st>>>(p);
        score_kernel<<<score_grid(p), 32 * kScoreQB, score_smem(p.D), st>>>(p);
        select_kernel<<<p.H * p.n_qb, 256, p.n_cand * sizeof(float), st>>>(p);
        lists_sparse_kernel<<<p.H * ((p.n_qb + 1) / 2), 128, 2 * ((p.n_cand + 31) / 32) * sizeof(uint32_t), st>>>(p);
    }
    return check_launch("mask_build kernels launch");
}

// ------------------------------------------------------------------------------------------------
// Allocation-free variant of the sparse selection: the pooled query / key means live in a
// file-scope device array instead of the caller's mask buffer.
// ------------------------------------------------------------------------------------------------
#include <mutex>

namespace nomas {

constexpr size_t kStaticPoolFloats = NOMAS_STATIC_POOL_FLOATS;   // 8 MiB of fp32 pooled means per device
static __device__ __align__(256) float g_pool_scratch[kStaticPoolFloats];

__global__ void qmean_to_kernel(MaskParams p, float *qmean) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n = (int64_t)p.H * p.n_qb * p.D;
    if (idx >= n) return;
    const int c = (int)(idx % p.D);
    const int64_t hb = idx / p.D;
    const int b = (int)(hb % p.n_qb);
    const int h = (int)(hb / p.n_qb);
    const int64_t r0 = (int64_t)b * kTile;
    const int nv = (int)((r0 + kTile < p.Nq) ? kTile : p.Nq - r0);
    float acc = 0.0f;
    for (int i = 0; i < nv; ++i)
        acc = __fadd_rn(acc, bf16_at(p.q, (r0 + i) * p.tok_stride + (int64_t)h * p.head_stride + c));
    qmean[idx] = __fdiv_rn(acc, (float)nv);
}

__global__ void kmean_to_kernel(MaskParams p, float *kmean) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.H * p.n_cand * p.D) return;
    kmean[idx] = kmean_value(p, idx);
}

__global__ void __launch_bounds__(32 * kScoreQB) score_from_kernel(MaskParams p, const float *qmean_all,
                                                                      const float *kmean_all) {
    score_block(p, qmean_all, kmean_all);
}

// Device address of this file's scratch array on the current device, looked up once per device.
static int static_pool_ptr(int device, float **out) {
    static std::mutex mu;
    static float *ptrs[256] = {};
    if (device < 0 || device >= 256) return NOMAS_EINVAL;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[device]) {
        void *ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_pool_scratch);
        if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(g_pool_scratch)", (int)e, cudaGetErrorString(e));
        ptrs[device] = static_cast<float *>(ptr);
    }
    *out = ptrs[device];
    return NOMAS_OK;
}

}  // namespace nomas

extern "C" int nomas_mask_build_static(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode,
                                       float keep_frac, const void *q, const void *kcur, int64_t tok_stride,
                                       int64_t head_stride, void *mask_buf, nomas_stream stream) {
    if (mode == NOMAS_MODE_DENSE)   // the dense build uses no scratch memory
        return nomas_mask_build(c, seg, mode, keep_frac, q, kcur, tok_stride, head_stride, mask_buf, stream);
    nomas_mask_layout lay;
    int rc = compute_mask_layout(c, seg, mode, keep_frac, &lay);
    if (rc) return rc;
    if (!mask_buf || !aligned16(mask_buf)) return NOMAS_EINVAL;
    if (!q || !kcur || !aligned16(q) || !aligned16(kcur)) return NOMAS_EINVAL;
    if (tok_stride <= 0 || head_stride <= 0 || tok_stride % 8 || head_stride % 8) return NOMAS_EINVAL;
    if (lay.n_cand < 1) return NOMAS_EINVAL;
    const size_t nq_floats = (size_t)c->d.heads * lay.n_qblocks * c->d.head_dim;
    const size_t nk_floats = (size_t)c->d.heads * lay.n_cand * c->d.head_dim;
    if (nq_floats + nk_floats > kStaticPoolFloats) return NOMAS_ECAPACITY;
    if (bind_device(c)) return NOMAS_ECUDA;
    float *pool = nullptr;
    rc = static_pool_ptr(c->device, &pool);
    if (rc) return rc;
    float *qmean = pool;
    float *kmean = pool + nq_floats;

    MaskParams p{};
    const HistView hv = hist_view(c);
    p.hdr.magic = kMaskMagic;
    p.hdr.mode = mode;
    p.hdr.n_qblocks = lay.n_qblocks;
    p.hdr.n_lists = lay.n_lists;
    p.hdr.history_tokens = lay.history_tokens;
    p.hdr.head_tokens = lay.head_tokens;
    p.hdr.frames_appended = c->frames_appended;
    p.hdr.n_query = lay.n_query;
    p.hdr.text_tokens = lay.text_tokens;
    p.hdr.list_cap = lay.list_cap;
    p.hdr.keep = lay.keep;
    p.n_tails = seg->n_tails;
    p.head_len = seg->head_len;
    for (int i = 0; i < seg->n_tails; ++i) p.tails[i] = seg->tails[i];
    p.T = c->d.tokens_per_frame;
    p.H = c->d.heads;
    p.D = c->d.head_dim;
    p.Lh = lay.history_tokens;
    p.Lp = lay.head_tokens;
    p.Nq = lay.n_query;
    p.Lt = lay.text_tokens;
    p.n_qb = lay.n_qblocks;
    p.n_tiles = lay.n_tiles;
    p.n_hist_tiles = lay.n_hist_tiles;
    p.n_head_tiles = lay.n_head_tiles;
    p.n_cur_tiles = lay.n_cur_tiles;
    p.n_text_tiles = lay.n_text_tiles;
    p.n_cand = lay.n_cand;
    p.keep = lay.keep;
    p.n_lists = lay.n_lists;
    p.list_cap = lay.list_cap;
    p.buf = static_cast<uint8_t *>(mask_buf);
    p.lay = lay;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.kcur = static_cast<const __nv_bfloat16 *>(kcur);
    p.tok_stride = tok_stride;
    p.head_stride = head_stride;
    p.k8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_K8]);
    p.ks = static_cast<const float *>(c->buf[NOMAS_BUF_KS]);
    p.ring_tokens = hv.ring_tokens;
    p.first_tok = hv.first_tok;

    // every pooled mean is written before it is read, so the shared array needs no clearing
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    mask_prep_kernel<<<nblk(lay.text_tokens > 0 ? lay.text_tokens : 1, 256), 256, 0, st>>>(p);
    class_map_kernel<<<nblk((int64_t)lay.n_qblocks * lay.n_tiles, 256), 256, 0, st>>>(p);
    qmean_to_kernel<<<nblk((int64_t)nq_floats, 256), 256, 0, st>>>(p, qmean);
    kmean_to_kernel<<<nblk((int64_t)nk_floats, 256), 256, 0, st>>>(p, kmean);
    score_from_kernel<<<score_grid(p), 32 * kScoreQB, score_smem(p.D), st>>>(p, qmean, kmean);
    select_kernel<<<p.H * p.n_qb, 256, p.n_cand * sizeof(float), st>>>(p);
    lists_sparse_kernel<<<p.H * ((p.n_qb + 1) / 2), 128, 2 * ((p.n_cand + 31) / 32) * sizeof(uint32_t), st>>>(p);
    return check_launch("mask_build_static kernels launch");
}
