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
//
// Launches: dense  mask_prep, class_map, lists_dense
//           sparse mask_prep, class_map, pool (block means), score, select_lists
//           text   mask_prep, class_map_text, lists_dense (query blocks of the current text)
#include <cmath>
#include <mutex>

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
    int *err;
    // sparse inputs
    const __nv_bfloat16 *q, *kcur;
    int64_t tok_stride, head_stride;
    const int8_t *k8;
    const float *ks;
    HistView hv;              // ring rows of the retained history in age order
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

// Text query blocks (NOMAS_MODE_TEXT): one CTA of 128 threads per (query block, KV tile), a thread per
// text row testing every key of the tile with the same visibility codes the attention kernel applies.
__device__ __forceinline__ VisCode key_code(const MaskParams &p, const TileInfo &ti, int k) {
    if (ti.kind == kKindCur) return key_video((int)((ti.start + k) / p.T));
    if (ti.kind == kKindText && ti.start + k >= p.head_len) {
        const int2 w = reinterpret_cast<const int2 *>(p.buf + p.lay.off_txtwin)[ti.start + k];
        return key_tail(w.x, w.y);
    }
    return key_always();
}

__global__ void __launch_bounds__(128) class_map_text_kernel(MaskParams p) {
    const int b = blockIdx.x / p.n_tiles, j = blockIdx.x % p.n_tiles;
    const TileInfo ti = tile_info(p, j);
    int8_t *cls = reinterpret_cast<int8_t *>(p.buf + p.lay.off_class) + (int64_t)b * p.n_tiles + j;
    if (ti.kind == kKindHist || ti.kind == kKindPriorHead) {   // always visible
        if (threadIdx.x == 0) *cls = 1;
        return;
    }
    const int64_t i = (int64_t)b * kTile + threadIdx.x;        // text row
    const bool row_ok = i < p.Lt;
    VisCode rc = row_head();
    if (row_ok && i >= p.head_len) {
        const int2 w = reinterpret_cast<const int2 *>(p.buf + p.lay.off_txtwin)[i];
        rc = row_tail(w.x, w.y);
    }
    int nvis = 0;
    if (row_ok)
        for (int k = 0; k < ti.count; ++k) nvis += visible(key_code(p, ti, k), rc) ? 1 : 0;
    const bool any = __syncthreads_or(row_ok && nvis > 0);
    const bool all = __syncthreads_and(!row_ok || nvis == ti.count);
    if (threadIdx.x == 0) *cls = all ? 1 : (any ? 2 : 0);
}

__device__ __forceinline__ int mask_flag(int8_t cls, int32_t count) { return (cls == 2 || count < kTile); }

// Dense lists: one warp per pair of query blocks (one attention CTA pair); lists are head-independent.
// Lanes test 32 tiles at a time and kept tiles are compacted in index order.
__global__ void lists_dense_kernel(MaskParams p) {
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

constexpr int kPoolAhead = 8;   // rows loaded before they are added (independent loads in flight)

// Block means.  Units [0, H*n_qb) are query blocks, then H*n_cand key candidates (history blocks in age
// order, then current-segment blocks); query and current-key units are numbered block-major (heads
// inner), so the consecutive units of a CTA read whole [tokens][heads][D] rows together.  A unit is
// handled by D/8 lanes, each summing 8 channels (one 16-byte load per row); a warp takes 32/(D/8)
// consecutive units.  Every channel is summed by one lane over
// the block's valid rows in ascending order from +0 (history keys as fp32(code) * scale, one rounding),
// then divided once by the number of valid rows.  Loads run kPoolAhead rows ahead of the additions,
// which keep the row order.
template <int D, bool CONTIG>
__global__ void __launch_bounds__(256) pool_kernel(MaskParams p, float *qmean, float *kmean) {
    constexpr int LPU = D / 8;             // lanes per unit
    constexpr int UPW = 32 / LPU;          // units per warp
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPU;
    const int64_t nq_units = (int64_t)p.H * p.n_qb;
    const int64_t n_units = nq_units + (int64_t)p.H * p.n_cand;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t ts = p.tok_stride;
    for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w * UPW < n_units; w += nwarps) {
        const int64_t u = w * UPW + lane / LPU;
        if (u >= n_units) continue;        // no warp-collective operation below
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        int nv;
        float *dst;
        bool hist = false;
        const __nv_bfloat16 *src = nullptr;
        int64_t h, r0;
        if (u < nq_units) {
            const int64_t b = u / p.H;
            h = u - b * p.H;
            r0 = b * (int64_t)kTile;
            nv = (int)(p.Nq - r0 < kTile ? p.Nq - r0 : kTile);
            src = p.q + r0 * ts + h * p.head_stride + sub * 8;
            dst = qmean + (h * p.n_qb + b) * D + sub * 8;
        } else {
            const int64_t v = u - nq_units;
            int cand;
            if (v < (int64_t)p.H * p.n_hist_tiles) {     // history: head-major (rows of a head are contiguous)
                h = v / p.n_hist_tiles;
                cand = (int)(v - h * p.n_hist_tiles);
            } else {                                     // current keys: block-major like the queries
                const int64_t w2 = v - (int64_t)p.H * p.n_hist_tiles;
                const int64_t b = w2 / p.H;
                h = w2 - b * p.H;
                cand = p.n_hist_tiles + (int)b;
            }
            dst = kmean + (h * p.n_cand + cand) * D + sub * 8;
            if (cand < p.n_hist_tiles) {
                hist = true;
                r0 = (int64_t)cand * kTile;
                nv = (int)(p.Lh - r0 < kTile ? p.Lh - r0 : kTile);
            } else {
                r0 = (int64_t)(cand - p.n_hist_tiles) * kTile;
                nv = (int)(p.Nq - r0 < kTile ? p.Nq - r0 : kTile);
                src = p.kcur + r0 * ts + h * p.head_stride + sub * 8;
            }
        }
        // full groups of kPoolAhead rows, then the remaining rows one at a time (same order)
        if (!hist) {
            auto add_row = [&](const uint4 &r) {
                const uint32_t wd[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[2 * c] = __fadd_rn(acc[2 * c], __uint_as_float(wd[c] << 16));
                    acc[2 * c + 1] = __fadd_rn(acc[2 * c + 1], __uint_as_float(wd[c] & 0xFFFF0000u));
                }
            };
            int i = 0;
            for (; i + kPoolAhead <= nv; i += kPoolAhead) {
                uint4 raw[kPoolAhead];
#pragma unroll
                for (int k = 0; k < kPoolAhead; ++k) {
                    raw[k] = __ldg(reinterpret_cast<const uint4 *>(src));
                    src += ts;
                }
#pragma unroll
                for (int k = 0; k < kPoolAhead; ++k) add_row(raw[k]);
            }
            for (; i < nv; ++i) {
                add_row(__ldg(reinterpret_cast<const uint4 *>(src)));
                src += ts;
            }
        } else {
            // ring rows of the block in age order; in a contiguous layout the physical row advances with
            // one wrap check, otherwise every row is looked up in the history map
            const int64_t ring = p.hv.ring_tokens;
            int64_t phys = hist_row(p.hv, r0);
            int64_t a = r0;
            auto next_row = [&]() {
                ++a;
                if (CONTIG) {
                    if (++phys == ring) phys = 0;
                } else if (a < r0 + nv) {
                    phys = hist_row(p.hv, a);
                }
            };
            const int8_t *kb = p.k8 + h * ring * D + sub * 8;
            const float *sb = p.ks + h * ring;
            auto add_row = [&](const uint2 &r, float sc) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t wd = c < 4 ? r.x : r.y;
                    acc[c] = __fadd_rn(acc[c], __fmul_rn((float)(int8_t)(wd >> (8 * (c & 3))), sc));
                }
            };
            int i = 0;
            for (; i + kPoolAhead <= nv; i += kPoolAhead) {
                uint2 raw[kPoolAhead];
                float sc[kPoolAhead];
#pragma unroll
                for (int k = 0; k < kPoolAhead; ++k) {
                    raw[k] = __ldg(reinterpret_cast<const uint2 *>(kb + phys * D));
                    sc[k] = __ldg(sb + phys);
                    next_row();
                }
#pragma unroll
                for (int k = 0; k < kPoolAhead; ++k) add_row(raw[k], sc[k]);
            }
            for (; i < nv; ++i) {
                add_row(__ldg(reinterpret_cast<const uint2 *>(kb + phys * D)), __ldg(sb + phys));
                next_row();
            }
        }
        const float n = (float)nv;
        float4 *d4 = reinterpret_cast<float4 *>(dst);
        d4[0] = make_float4(__fdiv_rn(acc[0], n), __fdiv_rn(acc[1], n), __fdiv_rn(acc[2], n), __fdiv_rn(acc[3], n));
        d4[1] = make_float4(__fdiv_rn(acc[4], n), __fdiv_rn(acc[5], n), __fdiv_rn(acc[6], n), __fdiv_rn(acc[7], n));
    }
}

// score[h][b][cand] = fmaf chain over channels in ascending order from +0.0f.  One CTA covers 64 query
// blocks x 64 candidates of one head; each of its 256 threads runs the 16 independent chains of a
// 4 x 4 patch.  Means are staged channel-major in shared memory, 64 channels at a time, so a thread
// reads its 4 query means and its 4 candidate means of one channel as two float4.
constexpr int kScoreTile = 64;

__global__ void __launch_bounds__(256) score_kernel(MaskParams p, const float *qmean, const float *kmean) {
    __shared__ __align__(16) float sq[64][kScoreTile];   // [channel in chunk][query block]
    __shared__ __align__(16) float sk[64][kScoreTile];   // [channel in chunk][candidate]
    const int D = p.D;
    const int h = blockIdx.y;
    const int n_ct = (p.n_cand + kScoreTile - 1) / kScoreTile;   // candidate tiles; x = qb tile * n_ct + ct
    const int b0 = (int)(blockIdx.x / n_ct) * kScoreTile, c0 = (int)(blockIdx.x % n_ct) * kScoreTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    const float *qm = qmean + (int64_t)h * p.n_qb * D;
    const float *km = kmean + (int64_t)h * p.n_cand * D;
    for (int ch0 = 0; ch0 < D; ch0 += 64) {
        __syncthreads();
        for (int i = threadIdx.x; i < kScoreTile * 16; i += blockDim.x) {
            const int r = i % kScoreTile, c4 = (i / kScoreTile) * 4;
            float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f), b = a;
            if (b0 + r < p.n_qb) a = *reinterpret_cast<const float4 *>(qm + (int64_t)(b0 + r) * D + ch0 + c4);
            if (c0 + r < p.n_cand) b = *reinterpret_cast<const float4 *>(km + (int64_t)(c0 + r) * D + ch0 + c4);
            sq[c4][r] = a.x;
            sq[c4 + 1][r] = a.y;
            sq[c4 + 2][r] = a.z;
            sq[c4 + 3][r] = a.w;
            sk[c4][r] = b.x;
            sk[c4 + 1][r] = b.y;
            sk[c4 + 2][r] = b.z;
            sk[c4 + 3][r] = b.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int c = 0; c < 64; ++c) {
            const float4 qv = *reinterpret_cast<const float4 *>(&sq[c][ty * 4]);
            const float4 kv = *reinterpret_cast<const float4 *>(&sk[c][tx * 4]);
            const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(qa[i], ka[j], acc[i][j]);
        }
    }
    float *sc = reinterpret_cast<float *>(p.buf + p.lay.off_score);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int b = b0 + ty * 4 + i;
        if (b >= p.n_qb) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cand = c0 + tx * 4 + j;
            if (cand < p.n_cand) sc[((int64_t)h * p.n_qb + b) * p.n_cand + cand] = acc[i][j];
        }
    }
}

// Ranking key with a total order: ascending key = score descending, then candidate index ascending.
// A NaN score ranks as -inf and -0 as +0, so every candidate has exactly one rank.
__device__ __forceinline__ unsigned long long rank_key(float s, int idx) {
    uint32_t u = __float_as_uint(s);
    if (s != s) u = 0xFF800000u;          // NaN -> -inf
    if (u == 0x80000000u) u = 0u;         // -0 -> +0
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // monotone in the float value
    return ((unsigned long long)(~ord) << 32) | (uint32_t)idx;
}

// One CTA per (head, pair of query blocks): the candidates of both query blocks are ranked at once
// (one bitonic sort per block over its keys, padded to npow2 with the largest key), the first `keep`
// of each are written to sel and marked in a bitmask, and warp 0 then writes the pair's tile list:
// kept candidates of either block in tile order, every earlier description head, and the text tiles
// by their dense class.
__global__ void __launch_bounds__(256) select_lists_kernel(MaskParams p, int npow2) {
    extern __shared__ unsigned long long keys[];                 // [2][npow2]
    uint32_t *bits = reinterpret_cast<uint32_t *>(keys + 2 * npow2);   // [2][words]
    const int n_pairs = (p.n_qb + 1) / 2;
    const int hp = blockIdx.x;           // h * n_pairs + pair
    const int h = hp / n_pairs, pr = hp % n_pairs;
    const int b0 = 2 * pr, b1 = 2 * pr + 1;
    const bool has1 = b1 < p.n_qb;
    const int words = (p.n_cand + 31) / 32;
    const float *sc = reinterpret_cast<const float *>(p.buf + p.lay.off_score);
    for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) bits[i] = 0;
    for (int i = threadIdx.x; i < 2 * npow2; i += blockDim.x) {
        const int seg = i / npow2, idx = i - seg * npow2;
        unsigned long long k = ~0ull;
        if (idx < p.n_cand && (seg == 0 || has1))
            k = rank_key(sc[((int64_t)h * p.n_qb + b0 + seg) * p.n_cand + idx], idx);
        keys[i] = k;
    }
    __syncthreads();
    // bitonic network on each npow2-long segment (pairs never cross a segment: j < npow2); j is a
    // power of two, so the pair index splits with a shift and a mask
    for (int k = 2; k <= npow2; k <<= 1) {
        for (int j = k >> 1, lj = __ffs(k) - 2; j > 0; j >>= 1, --lj) {
            for (int t = threadIdx.x; t < npow2; t += blockDim.x) {   // 2 * npow2 / 2 pairs
                const int e = ((t >> lj) << (lj + 1)) | (t & (j - 1));  // lower element, bit j clear
                const bool up = ((e & (npow2 - 1)) & k) == 0;
                const unsigned long long a = keys[e], b = keys[e + j];
                if ((a > b) == up) {
                    keys[e] = b;
                    keys[e + j] = a;
                }
            }
            __syncthreads();
        }
    }
    int32_t *sel = reinterpret_cast<int32_t *>(p.buf + p.lay.off_sel);
    for (int r = threadIdx.x; r < p.keep; r += blockDim.x) {
#pragma unroll
        for (int seg = 0; seg < 2; ++seg) {
            if (seg == 1 && !has1) continue;
            const uint32_t c = (uint32_t)keys[seg * npow2 + r];
            if (c >= (uint32_t)p.n_cand) {   // cannot happen (keep <= n_cand): record and skip
                set_device_error(p.err, NOMAS_EDEVICE, 20);
                continue;
            }
            sel[((int64_t)h * p.n_qb + b0 + seg) * p.keep + r] = (int32_t)c;
            atomicOr(&bits[seg * words + c / 32], 1u << (c % 32));
        }
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int8_t *cls = reinterpret_cast<const int8_t *>(p.buf + p.lay.off_class);
    int4 *out = reinterpret_cast<int4 *>(p.buf + p.lay.off_list) + (int64_t)hp * p.list_cap;
    int n = 0;
    for (int j0 = 0; j0 < p.n_tiles; j0 += 32) {
        const int j = j0 + lane;
        bool u0 = false, u1 = false, m0 = false, m1 = false;
        TileInfo ti{0, 0, 0};
        if (j < p.n_tiles) {
            ti = tile_info(p, j);
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
        }
        const bool keep = u0 || u1;
        const uint32_t m = __ballot_sync(0xffffffffu, keep);
        if (keep) {
            int f = ti.kind;
            if (u0) f |= kUse0 | (m0 ? kMask0 : 0);
            if (u1) f |= kUse1 | (m1 ? kMask1 : 0);
            out[n + __popc(m & ((1u << lane) - 1u))] = make_int4(f, (int)ti.start, ti.count, j);
        }
        n += __popc(m);
    }
    if (lane == 0) reinterpret_cast<int32_t *>(p.buf + p.lay.off_count)[hp] = n;
}

static unsigned nblk(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

static int pow2_at_least(int n) {
    int p = 2;
    while (p < n) p <<= 1;
    return p;
}

static size_t select_smem(int npow2, int n_cand) {
    return (size_t)2 * npow2 * sizeof(unsigned long long) + (size_t)2 * ((n_cand + 31) / 32) * sizeof(uint32_t);
}

// Validate the arguments of a mask build and fill the kernels' parameters (nothing is enqueued).
static int prepare_mask(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                        const void *q, const void *kcur, int64_t tok_stride, int64_t head_stride, void *mask_buf,
                        MaskParams &p) {
    nomas_mask_layout lay;
    const int rc = compute_mask_layout(c, seg, mode, keep_frac, &lay);
    if (rc) return rc;
    if (!mask_buf || !aligned16(mask_buf)) return NOMAS_EINVAL;
    if (mode == NOMAS_MODE_SPARSE) {
        if (!q || !kcur || !aligned16(q) || !aligned16(kcur)) return NOMAS_EINVAL;
        if (tok_stride <= 0 || head_stride <= 0 || tok_stride % 8 || head_stride % 8) return NOMAS_EINVAL;
        if (lay.n_cand < 1) return NOMAS_EINVAL;
    }
    const HistView hv = hist_view(c);
    p = MaskParams{};
    p.hdr.magic = kMaskMagic;
    p.hdr.mode = mode;
    p.hdr.n_qblocks = lay.n_qblocks;
    p.hdr.n_lists = lay.n_lists;
    p.hdr.history_tokens = lay.history_tokens;
    p.hdr.head_tokens = lay.head_tokens;
    p.hdr.cache_version = c->version;
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
    p.err = static_cast<int *>(c->buf[NOMAS_BUF_ERR]);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.kcur = static_cast<const __nv_bfloat16 *>(kcur);
    p.tok_stride = tok_stride;
    p.head_stride = head_stride;
    p.k8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_K8]);
    p.ks = static_cast<const float *>(c->buf[NOMAS_BUF_KS]);
    p.hv = hv;
    return NOMAS_OK;
}

// Raise the select kernel's dynamic shared-memory limit to what the largest supported candidate
// count needs (once per process; the attribute is per device function and the same on every device).
static int select_attr() {
    static std::once_flag once;
    static cudaError_t e = cudaSuccess;
    std::call_once(once, [] {
        e = cudaFuncSetAttribute(select_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)select_smem(pow2_at_least(NOMAS_MAX_SPARSE_CANDIDATES),
                                                  NOMAS_MAX_SPARSE_CANDIDATES));
    });
    return e == cudaSuccess ? NOMAS_OK : cuda_fail("cudaFuncSetAttribute(select smem)", (int)e, cudaGetErrorString(e));
}

// Enqueue the build.  qmean / kmean: where the sparse mode keeps its pooled means (scratch).
static int enqueue_mask(const MaskParams &p, float *qmean, float *kmean, cudaStream_t st) {
    const bool sp = p.hdr.mode == NOMAS_MODE_SPARSE;
    if (sp && select_attr()) return NOMAS_ECUDA;
    mask_prep_kernel<<<nblk(p.Lt > 0 ? p.Lt : 1, 256), 256, 0, st>>>(p);
    if (p.hdr.mode == NOMAS_MODE_TEXT) {
        class_map_text_kernel<<<(unsigned)((int64_t)p.n_qb * p.n_tiles), 128, 0, st>>>(p);
        lists_dense_kernel<<<nblk((int64_t)p.n_lists * 32, 128), 128, 0, st>>>(p);
        return check_launch("mask_build kernels launch");
    }
    class_map_kernel<<<nblk((int64_t)p.n_qb * p.n_tiles, 256), 256, 0, st>>>(p);
    if (!sp) {
        lists_dense_kernel<<<nblk((int64_t)p.n_lists * 32, 128), 128, 0, st>>>(p);
    } else {
        const int64_t units = (int64_t)p.H * (p.n_qb + p.n_cand);   // D/8 lanes each
        int64_t blocks = nblk(units * (p.D / 8), 256);
        if (blocks > 148 * 8) blocks = 148 * 8;
        const bool contig = p.hv.contiguous != 0;
        if (p.D == 128) {
            if (contig) pool_kernel<128, true><<<(unsigned)blocks, 256, 0, st>>>(p, qmean, kmean);
            else pool_kernel<128, false><<<(unsigned)blocks, 256, 0, st>>>(p, qmean, kmean);
        } else {
            if (contig) pool_kernel<64, true><<<(unsigned)blocks, 256, 0, st>>>(p, qmean, kmean);
            else pool_kernel<64, false><<<(unsigned)blocks, 256, 0, st>>>(p, qmean, kmean);
        }
        const dim3 sg(nblk(p.n_cand, kScoreTile) * nblk(p.n_qb, kScoreTile), (unsigned)p.H);
        score_kernel<<<sg, 256, 0, st>>>(p, qmean, kmean);
        const int npow2 = pow2_at_least(p.n_cand);
        select_lists_kernel<<<p.H * ((p.n_qb + 1) / 2), 256, select_smem(npow2, p.n_cand), st>>>(p, npow2);
    }
    return check_launch("mask_build kernels launch");
}

}  // namespace nomas

using namespace nomas;

extern "C" int nomas_mask_build(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                                const void *q, const void *kcur, int64_t tok_stride, int64_t head_stride,
                                void *mask_buf, nomas_stream stream) {
    MaskParams p;
    const int rc = prepare_mask(c, seg, mode, keep_frac, q, kcur, tok_stride, head_stride, mask_buf, p);
    if (rc) return rc;
    if (bind_device(c)) return NOMAS_ECUDA;
    uint8_t *mb = static_cast<uint8_t *>(mask_buf);
    return enqueue_mask(p, reinterpret_cast<float *>(mb + p.lay.off_qmean),
                        reinterpret_cast<float *>(mb + p.lay.off_kmean), reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------------------------------------
// Allocation-free variant of the sparse selection: the pooled query / key means live in a
// file-scope device array instead of the caller's mask buffer.
// ------------------------------------------------------------------------------------------------
namespace nomas {

constexpr size_t kStaticPoolFloats = NOMAS_STATIC_POOL_FLOATS;   // 8 MiB of fp32 pooled means per device
static __device__ __align__(256) float g_pool_scratch[kStaticPoolFloats];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// Device address of this file's scratch array in the calling thread's current context.  The address
// is looked up with cudaGetSymbolAddress the first time a context is seen and remembered per context,
// so a device whose primary context was reset (a new context) gets a fresh lookup.
static int static_pool_ptr(float **out) {
    static std::mutex mu;
    static CtxGetCurrentFn get_ctx = nullptr;
    static CUcontext ctxs[64] = {};
    static float *ptrs[64] = {};
    static int n = 0, next = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!get_ctx) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult qr = cudaDriverEntryPointSymbolNotFound;
        const cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &qr);
        if (e != cudaSuccess || qr != cudaDriverEntryPointSuccess)
            return cuda_fail("cudaGetDriverEntryPoint(cuCtxGetCurrent)", e != cudaSuccess ? (int)e : (int)qr,
                             "symbol query failed");
        get_ctx = reinterpret_cast<CtxGetCurrentFn>(fn);
    }
    CUcontext ctx = nullptr;
    const CUresult cr = get_ctx(&ctx);
    if (cr != CUDA_SUCCESS || !ctx) return cuda_fail("cuCtxGetCurrent", (int)cr, "no current context");
    for (int i = 0; i < n; ++i)
        if (ctxs[i] == ctx) {
            *out = ptrs[i];
            return NOMAS_OK;
        }
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_pool_scratch);
    if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(g_pool_scratch)", (int)e, cudaGetErrorString(e));
    const int slot = n < 64 ? n++ : (next++ % 64);   // remember the most recent 64 contexts
    ctxs[slot] = ctx;
    ptrs[slot] = static_cast<float *>(ptr);
    *out = ptrs[slot];
    return NOMAS_OK;
}

}  // namespace nomas

extern "C" int nomas_mask_build_static(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode,
                                       float keep_frac, const void *q, const void *kcur, int64_t tok_stride,
                                       int64_t head_stride, void *mask_buf, nomas_stream stream) {
    if (mode == NOMAS_MODE_DENSE)   // the dense build uses no scratch memory
        return nomas_mask_build(c, seg, mode, keep_frac, q, kcur, tok_stride, head_stride, mask_buf, stream);
    MaskParams p;
    int rc = prepare_mask(c, seg, mode, keep_frac, q, kcur, tok_stride, head_stride, mask_buf, p);
    if (rc) return rc;
    const size_t nq_floats = (size_t)c->d.heads * p.n_qb * c->d.head_dim;
    const size_t nk_floats = (size_t)c->d.heads * p.n_cand * c->d.head_dim;
    if (nq_floats + nk_floats > kStaticPoolFloats) return NOMAS_ECAPACITY;
    if (bind_device(c)) return NOMAS_ECUDA;
    float *pool = nullptr;
    rc = static_pool_ptr(&pool);
    if (rc) return rc;
    // every pooled mean is written before it is read, so the shared array needs no clearing
    return enqueue_mask(p, pool, pool + nq_floats, reinterpret_cast<cudaStream_t>(stream));
}
