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
//           sparse mask_prep, class_map, pool (block means, TMA-fed), score, select_lists
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
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
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

// Video query blocks: SKIP / FULL / PARTIAL per (query block, KV tile) over valid rows and valid keys.
// History, earlier heads and current video are visible to every video row, so those tiles are FULL;
// blocks [0, plain_blocks) write them, one thread per entry.  The remaining blocks give one warp to
// each (query block, text tile): lanes hold the windows of 4 keys each and, frame by frame over the
// block's rows, count the keys visible to that frame.
__global__ void class_map_kernel(MaskParams p, int plain_blocks) {
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
    int8_t *cls = reinterpret_cast<int8_t *>(p.buf + p.lay.off_class);
    const int n_plain = p.n_tiles - p.n_text_tiles;      // text tiles come last in tile order
    if ((int)blockIdx.x < plain_blocks) {
        const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        if (idx >= (int64_t)p.n_qb * n_plain) return;
        const int64_t b = idx / n_plain;
        cls[b * p.n_tiles + (idx - b * n_plain)] = 1;
        return;
    }
    const int64_t wi = ((int64_t)(blockIdx.x - plain_blocks) * blockDim.x + threadIdx.x) >> 5;
    if (wi >= (int64_t)p.n_qb * p.n_text_tiles) return;  // warp-uniform
    const int lane = threadIdx.x & 31;
    const int b = (int)(wi / p.n_text_tiles), j = n_plain + (int)(wi - (int64_t)b * p.n_text_tiles);
    const TileInfo ti = tile_info(p, j);
    const int2 *win = reinterpret_cast<const int2 *>(p.buf + p.lay.off_txtwin);
    int2 w[kTile / 32];
#pragma unroll
    for (int i = 0; i < kTile / 32; ++i) {
        const int k = lane + 32 * i;
        w[i] = k < ti.count ? win[ti.start + k] : make_int2(0, 0);   // an absent key is never visible
    }
    const int64_t r0 = (int64_t)b * kTile;
    const int64_t r1 = (r0 + kTile < p.Nq) ? r0 + kTile : p.Nq;
    int64_t vis = 0;
    for (int64_t t = r0 / p.T; t <= (r1 - 1) / p.T; ++t) {
        int nk = 0;
#pragma unroll
        for (int i = 0; i < kTile / 32; ++i) nk += (w[i].x <= t && t < w[i].y) ? 1 : 0;
        nk = __reduce_add_sync(0xffffffffu, nk);
        const int64_t a0 = t * p.T > r0 ? t * p.T : r0;
        const int64_t a1 = (t + 1) * p.T < r1 ? (t + 1) * p.T : r1;
        vis += (a1 - a0) * nk;
    }
    const int64_t total = (r1 - r0) * ti.count;
    if (lane == 0) cls[(int64_t)b * p.n_tiles + j] = vis == total ? 1 : (vis == 0 ? 0 : 2);
}

// Text query blocks (NOMAS_MODE_TEXT): one CTA of 128 threads per (query block, KV tile), a thread per
// text row, with the visibility codes the attention kernel applies.  History and earlier heads are
// visible to every text row.  Current video: a head row sees every frame, a tail row the frames of its
// window, so the count is an interval overlap.  Text keys: their codes are staged in shared memory and
// every row tests each.
__device__ __forceinline__ VisCode text_key_code(const MaskParams &p, int64_t i) {
    if (i < p.head_len) return key_always();
    const int2 w = reinterpret_cast<const int2 *>(p.buf + p.lay.off_txtwin)[i];
    return key_tail(w.x, w.y);
}

__global__ void __launch_bounds__(128) class_map_text_kernel(MaskParams p) {
    __shared__ VisCode skey[kTile];
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
    const int b = blockIdx.x / p.n_tiles, j = blockIdx.x % p.n_tiles;
    const TileInfo ti = tile_info(p, j);
    int8_t *cls = reinterpret_cast<int8_t *>(p.buf + p.lay.off_class) + (int64_t)b * p.n_tiles + j;
    if (ti.kind == kKindHist || ti.kind == kKindPriorHead) {   // always visible
        if (threadIdx.x == 0) *cls = 1;
        return;
    }
    const int64_t i = (int64_t)b * kTile + threadIdx.x;        // text row
    const bool row_ok = i < p.Lt;
    const bool tail_row = row_ok && i >= p.head_len;
    const int2 rw = tail_row ? reinterpret_cast<const int2 *>(p.buf + p.lay.off_txtwin)[i] : make_int2(0, 0);
    int nvis = 0;
    if (ti.kind == kKindCur) {                                  // block-uniform branch
        if (row_ok && !tail_row) {
            nvis = ti.count;
        } else if (tail_row) {
            const int64_t lo = (int64_t)rw.x * p.T > ti.start ? (int64_t)rw.x * p.T : ti.start;
            const int64_t hi = (int64_t)rw.y * p.T < ti.start + ti.count ? (int64_t)rw.y * p.T : ti.start + ti.count;
            nvis = hi > lo ? (int)(hi - lo) : 0;
        }
    } else {
        skey[threadIdx.x] = (int)threadIdx.x < ti.count ? text_key_code(p, ti.start + threadIdx.x) : key_none();
        __syncthreads();
        if (row_ok) {
            const VisCode rc = tail_row ? row_tail(rw.x, rw.y) : row_head();
            for (int k = 0; k < ti.count; ++k) nvis += visible(skey[k], rc) ? 1 : 0;
        }
    }
    const bool any = __syncthreads_or(row_ok && nvis > 0);
    const bool all = __syncthreads_and(!row_ok || nvis == ti.count);
    if (threadIdx.x == 0) *cls = all ? 1 : (any ? 2 : 0);
}

__device__ __forceinline__ int mask_flag(int8_t cls, int32_t count) { return (cls == 2 || count < kTile); }

// Dense lists: one warp per pair of query blocks (one attention CTA pair); lists are head-independent.
// Lanes test 32 tiles at a time and kept tiles are compacted in index order.
__global__ void lists_dense_kernel(MaskParams p) {
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
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

// Block means, fed by TMA.  A persistent kernel: per CTA a producer warp streams the rows of its units
// into a three-stage shared-memory ring while four consumer warps add them.  A unit is one 128-row block
// of one head group (1024 / D heads, so that each of the 128 consumer threads sums 8 channels of one
// head): a query block, a current-key block (both one tensor-map box of R rows x heads x D per stage),
// or a history tile (per head, untiled bulk copies of each run of consecutive ring rows of the INT8
// codes, and of the 16-byte-aligned span of their scales, 16 rows per stage).  Every channel is summed
// by one thread over the block's valid rows in ascending order from +0 (history keys as fp32(code) *
// scale, one rounding), then divided once by the number of valid rows.  Units are dealt to CTAs
// round-robin, blocks of q and current keys first.
constexpr int kPoolRows = 16;       // rows per stage (bf16 stages: min(16, query rows))
constexpr int kPoolStages = 2;     // with three CTAs per SM (measured best of 1-3 CTAs x 2-6 stages)
constexpr int kPoolConsumers = 4;   // warps; warp 4 is the producer
constexpr int kPoolThreads = 32 * (kPoolConsumers + 1);

template <int D>
struct PoolCfg {
    static constexpr int HG = 1024 / D;                          // heads per unit
    static constexpr int STAGE = kPoolRows * HG * D * 2;         // 32 KB
    static constexpr int SC_SLOTS = 128;                         // scale slots per head and history stage
    static constexpr int OFF_SC = kPoolRows * HG * D;            // history: fp32 [HG][SC_SLOTS] after the codes
    static constexpr int OFF_IDX = OFF_SC + HG * SC_SLOTS * 4;   // uint8 [HG][16]: row -> scale slot
    static constexpr int OFF_BAR = kPoolStages * STAGE;
    static constexpr int SMEM = OFF_BAR + 2 * kPoolStages * 8 + 128;   // + slack for 128-byte alignment
    static_assert(OFF_IDX + HG * kPoolRows <= STAGE, "a history stage fits in a stage");
};

struct PoolParams {
    int32_t R;          // rows of a q / current-key box: min(16, query rows)
    int32_t HGb;        // heads of a box: min(heads per unit, H)
    int32_t n_hg;       // head groups
    int64_t n_units;
    float *qmean, *kmean;
    uint64_t timeout_ns;
};

struct PoolUnit {
    int kind;           // 0 query block, 1 current-key block, 2 history tile
    int blk;
    int g;              // head group
    int nv;             // valid rows
};

__device__ __forceinline__ PoolUnit pool_unit(const MaskParams &p, const PoolParams &pp, int64_t u) {
    PoolUnit r;
    const int64_t nb = (int64_t)2 * p.n_qb * pp.n_hg;
    int64_t rem;
    if (u < nb) {                                   // head group fastest, then q / k, then block
        const int64_t t = u / pp.n_hg;
        r.g = (int)(u - t * pp.n_hg);
        r.kind = (int)(t & 1);
        r.blk = (int)(t >> 1);
        rem = p.Nq - (int64_t)r.blk * kTile;
    } else {
        const int64_t v = u - nb, t = v / pp.n_hg;
        r.g = (int)(v - t * pp.n_hg);
        r.kind = 2;
        r.blk = (int)t;
        rem = p.Lh - (int64_t)r.blk * kTile;
    }
    r.nv = rem < kTile ? (int)rem : kTile;
    return r;
}

// One run of consecutive ring rows of the history, starting at age a: its physical row and length
// (at most `left`; it ends at the ring's end or, in a slot table, at the frame's end).
__device__ __forceinline__ int hist_run(const HistView &hv, int64_t a, int left, int64_t &phys) {
    int64_t room;
    if (hv.contiguous) {
        phys = hv.first_tok + a;
        if (phys >= hv.ring_tokens) phys -= hv.ring_tokens;
        room = hv.ring_tokens - phys;
    } else {
        const int64_t f = a / hv.T, o = a - f * hv.T;
        phys = (int64_t)hv.slots[f] * hv.T + o;
        room = hv.T - o;
    }
    return room < left ? (int)room : left;
}

// Producer side of one history stage (rows a0 .. a0 + n - 1 of every head of group g): lane l < HGb copies
// head g * HG + l.  The transaction count is raised by the total first, then the copies are issued and
// the row -> scale-slot map is written, and lane 0 arrives once everything is issued.
template <int D>
__device__ __forceinline__ void hist_stage(const MaskParams &p, const PoolParams &pp, const PoolUnit &un, int s,
                                           uint8_t *buf, uint64_t *bar, int lane) {
    using C = PoolCfg<D>;
    const int64_t a0 = (int64_t)un.blk * kTile + s * kPoolRows;
    const int n = un.nv - s * kPoolRows < kPoolRows ? un.nv - s * kPoolRows : kPoolRows;
    const int h = un.g * pp.HGb + lane;
    const bool act = lane < pp.HGb && h < p.H;
    const int64_t hbase = (int64_t)h * p.hv.ring_tokens;
    uint32_t bytes = 0;
    if (act) {
        int64_t a = a0;
        for (int left = n; left > 0;) {
            int64_t phys;
            const int len = hist_run(p.hv, a, left, phys);
            const int64_t i0 = hbase + phys;
            bytes += (uint32_t)(len * D) + (uint32_t)((((i0 + len + 3) & ~3ll) - (i0 & ~3ll)) * 4);
            a += len;
            left -= len;
        }
    }
    bytes = __reduce_add_sync(0xffffffffu, bytes);
    if (lane == 0) mbar_expect_tx(bar, bytes);
    __syncwarp();
    if (act) {
        uint8_t *idx = buf + C::OFF_IDX + lane * kPoolRows;
        int64_t a = a0;
        int r = 0, pos = 0;
        for (int left = n; left > 0;) {
            int64_t phys;
            const int len = hist_run(p.hv, a, left, phys);
            const int64_t i0 = hbase + phys, lo = i0 & ~3ll, hi = (i0 + len + 3) & ~3ll;
            bulk_load(buf + (lane * kPoolRows + r) * D, p.k8 + i0 * D, (uint32_t)(len * D), bar);
            bulk_load(buf + C::OFF_SC + (lane * C::SC_SLOTS + pos) * 4, p.ks + lo, (uint32_t)((hi - lo) * 4), bar);
            for (int t = 0; t < len; ++t) idx[r + t] = (uint8_t)(pos + (int)(i0 - lo) + t);
            pos += (int)(hi - lo);
            r += len;
            a += len;
            left -= len;
        }
        fence_proxy_async_smem();   // the map's generic stores before later async copies into this stage
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __grid_constant__ CUtensorMap tq,
                                                            const __grid_constant__ CUtensorMap tk,
                                                            const __grid_constant__ MaskParams p,
                                                            const PoolParams pp) {
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
    using C = PoolCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 127u) & ~127u) - raw_addr);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR), *empty = full + kPoolStages;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPoolStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kPoolConsumers);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    Watchdog wd{p.err, &abort_flag, pp.timeout_ns, 8};
    const uint32_t box_bytes = (uint32_t)(pp.R * pp.HGb * D * 2);

    if (warp == kPoolConsumers) {
        // ---------------------------------------------------------------- producer warp
        uint32_t issued = 0, par = 0;     // per stage: copies issued, parity of the phase they complete
        int i = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < pp.n_units && ok; u += gridDim.x) {
            const PoolUnit un = pool_unit(p, pp, u);
            const int rows = un.kind == 2 ? kPoolRows : pp.R;
            const int ns = (un.nv + rows - 1) / rows;
            for (int s = 0; s < ns; ++s, ++i) {
                const int st = i % kPoolStages;
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ((i / kPoolStages) & 1) ^ 1, wd, 1))) {
                    ok = false;
                    break;
                }
                uint8_t *buf = sm + st * C::STAGE;
                if (un.kind != 2) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[st], box_bytes);
                        tma_load_3d(buf, un.kind ? &tk : &tq, &full[st], 0, un.g * pp.HGb, un.blk * kTile + s * pp.R);
                    }
                } else {
                    hist_stage<D>(p, pp, un, s, buf, &full[st], lane);
                }
                issued |= 1u << st;
                par = (par & ~(1u << st)) | ((uint32_t)((i / kPoolStages) & 1) << st);
            }
        }
        // copies in flight must land before the CTA's shared memory is released (a no-op unless aborting)
        if (lane == 0)
            for (int st = 0; st < kPoolStages; ++st)
                if ((issued >> st) & 1u) mbar_drain(&full[st], (par >> st) & 1u, 100000000ull);
        return;
    }
    // -------------------------------------------------------------------- consumers
    const int t = threadIdx.x;               // 0 .. 127
    const int hl = t / (D / 8), sub = t % (D / 8);
    int i = 0;
    for (int64_t u = blockIdx.x; u < pp.n_units; u += gridDim.x) {
        const PoolUnit un = pool_unit(p, pp, u);
        const int rows = un.kind == 2 ? kPoolRows : pp.R;
        const int ns = (un.nv + rows - 1) / rows;
        const int h = un.g * pp.HGb + hl;
        const bool head_ok = hl < pp.HGb && h < p.H;     // this thread's head was copied
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
        bool ok = true;
        for (int s = 0; s < ns; ++s, ++i) {
            const int st = i % kPoolStages;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (i / kPoolStages) & 1, wd, 2))) {
                ok = false;
                break;
            }
            const int n = un.nv - s * rows < rows ? un.nv - s * rows : rows;
            const uint8_t *buf = sm + st * C::STAGE;
            if (head_ok && un.kind != 2) {
                const uint4 *src = reinterpret_cast<const uint4 *>(buf + ((size_t)hl * D + sub * 8) * 2);
                const int step = pp.HGb * D / 8;   // uint4 per box row
#pragma unroll 4
                for (int r = 0; r < n; ++r) {
                    const uint4 w = src[r * step];
                    const uint32_t wd4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        acc[2 * c] = __fadd_rn(acc[2 * c], __uint_as_float(wd4[c] << 16));
                        acc[2 * c + 1] = __fadd_rn(acc[2 * c + 1], __uint_as_float(wd4[c] & 0xFFFF0000u));
                    }
                }
            } else if (head_ok) {
                const uint8_t *cb = buf + hl * kPoolRows * D + sub * 8;
                const float *scb = reinterpret_cast<const float *>(buf + C::OFF_SC) + hl * C::SC_SLOTS;
                const uint8_t *ib = buf + C::OFF_IDX + hl * kPoolRows;
#pragma unroll 4
                for (int r = 0; r < n; ++r) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(cb + r * D);
                    const float sc = scb[ib[r]];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t wd = c < 4 ? w.x : w.y;
                        acc[c] = __fadd_rn(acc[c], __fmul_rn((float)(int8_t)(wd >> (8 * (c & 3))), sc));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (!ok) break;
        if (!head_ok) continue;
        float *dst;
        if (un.kind == 0) dst = pp.qmean + ((int64_t)h * p.n_qb + un.blk) * D;
        else if (un.kind == 1) dst = pp.kmean + ((int64_t)h * p.n_cand + p.n_hist_tiles + un.blk) * D;
        else dst = pp.kmean + ((int64_t)h * p.n_cand + un.blk) * D;
        const float nvf = (float)un.nv;
        float4 *d4 = reinterpret_cast<float4 *>(dst + sub * 8);
        d4[0] = make_float4(__fdiv_rn(acc[0], nvf), __fdiv_rn(acc[1], nvf), __fdiv_rn(acc[2], nvf), __fdiv_rn(acc[3], nvf));
        d4[1] = make_float4(__fdiv_rn(acc[4], nvf), __fdiv_rn(acc[5], nvf), __fdiv_rn(acc[6], nvf), __fdiv_rn(acc[7], nvf));
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
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
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

// The tile list of one attention CTA pair (head h, query blocks 2 pr and 2 pr + 1), written by one warp:
// kept candidates of either block (bit masks bits0, bits1; bits1 null when the pair has one block) in
// tile order, every earlier description head, and the text tiles by their dense class.
__device__ void write_pair_list(const MaskParams &p, int h, int pr, const uint32_t *bits0, const uint32_t *bits1,
                                int lane) {
    const int n_pairs = (p.n_qb + 1) / 2;
    const int hp = h * n_pairs + pr;
    const int b0 = 2 * pr, b1 = 2 * pr + 1;
    const bool has1 = bits1 != nullptr;
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
                u0 = (bits0[cand / 32] >> (cand % 32)) & 1u;
                u1 = has1 && ((bits1[cand / 32] >> (cand % 32)) & 1u);
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

// Bitonic networks over the 32 M keys of a warp, element e = lane * M + i (lane l holds elements
// l M .. l M + M - 1): partners at distance j >= M are exchanged across lanes by shuffles, closer ones
// inside the lane.  warp_sort_up sorts ascending; warp_merge_up sorts a bitonic sequence ascending.
template <int M>
__device__ __forceinline__ void warp_sort_up(unsigned long long (&a)[M], int lane) {
    for (int k = 2; k <= 32 * M; k <<= 1) {
        for (int j = k >> 1; j >= M; j >>= 1) {            // partner in lane ^ (j / M), same register
            const int lm = j / M;
            const bool take_min = ((lane & lm) == 0) == (((lane * M) & k) == 0);
#pragma unroll
            for (int i = 0; i < M; ++i) {
                const unsigned long long o = __shfl_xor_sync(0xffffffffu, a[i], lm);
                a[i] = take_min ? (o < a[i] ? o : a[i]) : (o > a[i] ? o : a[i]);
            }
        }
#pragma unroll
        for (int j = M / 2; j > 0; j >>= 1) {               // partner in the same lane
            if (j >= k) continue;
#pragma unroll
            for (int i = 0; i < M; ++i) {
                if (i & j) continue;
                const bool up = ((lane * M + i) & k) == 0;
                const unsigned long long x = a[i], y = a[i ^ j];
                const bool sw = (x > y) == up;
                a[i] = sw ? y : x;
                a[i ^ j] = sw ? x : y;
            }
        }
    }
}

template <int M>
__device__ __forceinline__ void warp_merge_up(unsigned long long (&a)[M], int lane) {
#pragma unroll
    for (int j = 16 * M; j >= M; j >>= 1) {
        const int lm = j / M;
        const bool take_min = (lane & lm) == 0;
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, a[i], lm);
            a[i] = take_min ? (o < a[i] ? o : a[i]) : (o > a[i] ? o : a[i]);
        }
    }
#pragma unroll
    for (int j = M / 2; j > 0; j >>= 1) {
#pragma unroll
        for (int i = 0; i < M; ++i) {
            if (i & j) continue;
            const unsigned long long x = a[i], y = a[i ^ j];
            a[i] = x < y ? x : y;
            a[i ^ j] = x < y ? y : x;
        }
    }
}

// Selection when keep <= 128: one warp per query block keeps the 128 smallest keys (ascending) of the
// candidates seen so far.  Candidates arrive in chunks of 128 (4 per lane, padded with the largest key);
// a chunk is sorted, and with B its sorted keys the 128 smallest of A and B are min(A[e], B[127 - e]),
// a bitonic sequence that one merge network sorts.  The first `keep` keys are the kept candidates in
// rank order -- the same result as sorting every key.  Then warps 0..3 write the CTA's pair lists.
__global__ void __launch_bounds__(256, 4) select_lists_top128_kernel(MaskParams p) {
    __shared__ uint32_t bits[8][32];             // kept-candidate bit mask per query block (1024 bits)
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
    const int n_pairs = (p.n_qb + 1) / 2;
    const int groups = (n_pairs + 3) / 4;
    const int h = blockIdx.x / groups, g = blockIdx.x - h * groups;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = 8 * g + warp;
    const bool valid = b < p.n_qb;
    uint32_t *bw = bits[warp];
    unsigned long long a[4];
    const float *sc = reinterpret_cast<const float *>(p.buf + p.lay.off_score) + ((int64_t)h * p.n_qb + b) * p.n_cand;
    for (int c0 = 0; c0 < p.n_cand; c0 += 128) {
        unsigned long long t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = c0 + lane * 4 + i;
            t[i] = (valid && c < p.n_cand) ? rank_key(sc[c], c) : ~0ull;
        }
        warp_sort_up<4>(t, lane);
        if (c0 == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = t[i];
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const unsigned long long o = __shfl_xor_sync(0xffffffffu, t[3 - i], 31);   // B[127 - e]
                a[i] = o < a[i] ? o : a[i];
            }
            warp_merge_up<4>(a, lane);
        }
    }
    bw[lane] = 0;
    __syncwarp();
    if (valid) {
        int32_t *sel = reinterpret_cast<int32_t *>(p.buf + p.lay.off_sel) + ((int64_t)h * p.n_qb + b) * p.keep;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = lane * 4 + i;
            if (r >= p.keep) continue;
            const uint32_t c = (uint32_t)a[i];
            if (c >= (uint32_t)p.n_cand) {                  // cannot happen (keep <= n_cand): record and skip
                set_device_error(p.err, NOMAS_EDEVICE, 20);
                continue;
            }
            sel[r] = (int32_t)c;
            atomicOr(&bw[c >> 5], 1u << (c & 31));
        }
    }
    __syncthreads();
    const int pr = 4 * g + warp;
    if (warp < 4 && pr < n_pairs)
        write_pair_list(p, h, pr, bits[2 * warp], 2 * pr + 1 < p.n_qb ? bits[2 * warp + 1] : nullptr, lane);
}

// Selection with the keys in registers: one warp per query block (eight per CTA, four CTA pairs), up to
// 32 M candidates, M keys per lane.  Lane l starts with candidates i * 32 + l (the order does not matter:
// every key carries its index) and the bitonic network runs on element e = l M + i, exchanging across
// lanes by shuffles when the partner distance is M or more and inside the lane otherwise.  The first
// `keep` elements of the ascending order are the kept candidates in rank order; then warps 0..3 write
// the lists of the CTA's pairs.
template <int M>
__global__ void __launch_bounds__(256, M >= 32 ? 1 : 2) select_lists_warp_kernel(MaskParams p) {
    __shared__ uint32_t bits[8][M];            // kept-candidate bit mask per query block (32 M bits)
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
    const int n_pairs = (p.n_qb + 1) / 2;
    const int groups = (n_pairs + 3) / 4;
    const int h = blockIdx.x / groups, g = blockIdx.x - h * groups;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = 8 * g + warp;                  // = 2 * (4 g + warp / 2) + warp % 2
    const bool valid = b < p.n_qb;
    if (lane < M) bits[warp][lane] = 0;
    unsigned long long a[M];
    const float *sc = reinterpret_cast<const float *>(p.buf + p.lay.off_score) + ((int64_t)h * p.n_qb + b) * p.n_cand;
#pragma unroll
    for (int i = 0; i < M; ++i) {
        const int c = i * 32 + lane;
        a[i] = (valid && c < p.n_cand) ? rank_key(sc[c], c) : ~0ull;
    }
    warp_sort_up<M>(a, lane);
    __syncwarp();
    if (valid) {
        int32_t *sel = reinterpret_cast<int32_t *>(p.buf + p.lay.off_sel) + ((int64_t)h * p.n_qb + b) * p.keep;
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const int r = lane * M + i;
            if (r >= p.keep) continue;
            const uint32_t c = (uint32_t)a[i];
            if (c >= (uint32_t)p.n_cand) {                  // cannot happen (keep <= n_cand): record and skip
                set_device_error(p.err, NOMAS_EDEVICE, 20);
                continue;
            }
            sel[r] = (int32_t)c;
            atomicOr(&bits[warp][c >> 5], 1u << (c & 31));
        }
    }
    __syncthreads();
    const int pr = 4 * g + warp;
    if (warp < 4 && pr < n_pairs)
        write_pair_list(p, h, pr, bits[2 * warp], 2 * pr + 1 < p.n_qb ? bits[2 * warp + 1] : nullptr, lane);
}

// One CTA per (head, pair of query blocks): the candidates of both query blocks are ranked at once
// (one bitonic sort per block over its keys, padded to npow2 with the largest key), the first `keep`
// of each are written to sel and marked in a bitmask, and warp 0 then writes the pair's tile list:
// kept candidates of either block in tile order, every earlier description head, and the text tiles
// by their dense class.
__global__ void __launch_bounds__(256) select_lists_kernel(MaskParams p, int npow2) {
    extern __shared__ unsigned long long keys[];                 // [2][npow2]
    uint32_t *bits = reinterpret_cast<uint32_t *>(keys + 2 * npow2);   // [2][words]
    griddep_wait();   // the previous grid of the stream has completed (programmatic launch)
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
    if (threadIdx.x < 32) write_pair_list(p, h, pr, bits, has1 ? bits + words : nullptr, threadIdx.x);
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

// Raise the dynamic shared-memory limits of the select kernel (to what the largest supported candidate
// count needs) and of the pooling kernels (once per process; the attribute is per device function and
// the same on every device).
static int kernel_attrs() {
    static std::once_flag once;
    static cudaError_t e = cudaSuccess;
    std::call_once(once, [] {
        e = cudaFuncSetAttribute(select_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)select_smem(pow2_at_least(NOMAS_MAX_SPARSE_CANDIDATES),
                                                  NOMAS_MAX_SPARSE_CANDIDATES));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(pool_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, PoolCfg<128>::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(pool_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, PoolCfg<64>::SMEM);
    });
    return e == cudaSuccess ? NOMAS_OK : cuda_fail("cudaFuncSetAttribute(mask kernels smem)", (int)e, cudaGetErrorString(e));
}

// Enqueue the build.  qmean / kmean: where the sparse mode keeps its pooled means (scratch).
static int enqueue_mask(const MaskParams &p, float *qmean, float *kmean, cudaStream_t st) {
    const bool sp = p.hdr.mode == NOMAS_MODE_SPARSE;
    // the pooling kernel's tensor maps and parameters first, so that a failure enqueues nothing
    CUtensorMap tq, tk;
    PoolParams pp{};
    if (sp) {
        if (kernel_attrs()) return NOMAS_ECUDA;
        const int hg = 1024 / p.D;
        pp.HGb = p.H < hg ? p.H : hg;
        pp.R = p.Nq < kPoolRows ? (int)p.Nq : kPoolRows;
        pp.n_hg = (p.H + pp.HGb - 1) / pp.HGb;
        pp.n_units = (int64_t)pp.n_hg * (2 * (int64_t)p.n_qb + p.n_hist_tiles);
        pp.qmean = qmean;
        pp.kmean = kmean;
        pp.timeout_ns = wait_limit_ns();
        const cuuint64_t dims[3] = {(cuuint64_t)p.D, (cuuint64_t)p.H, (cuuint64_t)p.Nq};
        const cuuint64_t strides[2] = {(cuuint64_t)p.head_stride * 2, (cuuint64_t)p.tok_stride * 2};
        const cuuint32_t box[3] = {(cuuint32_t)p.D, (cuuint32_t)pp.HGb, (cuuint32_t)pp.R};
        if (!make_tensor_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !make_tensor_map_3d(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.kcur, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
            return NOMAS_ECUDA;
    }
    launch_pdl(mask_prep_kernel, nblk(p.Lt > 0 ? p.Lt : 1, 256), 256, 0, st, p);
    if (p.hdr.mode == NOMAS_MODE_TEXT) {
        launch_pdl(class_map_text_kernel, (unsigned)((int64_t)p.n_qb * p.n_tiles), 128, 0, st, p);
        launch_pdl(lists_dense_kernel, nblk((int64_t)p.n_lists * 32, 128), 128, 0, st, p);
        return check_launch("mask_build kernels launch");
    }
    {
        const unsigned plain = nblk((int64_t)p.n_qb * (p.n_tiles - p.n_text_tiles), 256);
        const unsigned text = nblk((int64_t)p.n_qb * p.n_text_tiles * 32, 256);
        if (plain + text > 0) launch_pdl(class_map_kernel, plain + text, 256, 0, st, p, (int)plain);
    }
    if (!sp) {
        launch_pdl(lists_dense_kernel, nblk((int64_t)p.n_lists * 32, 128), 128, 0, st, p);
    } else {
        int64_t blocks = (int64_t)3 * sm_count();     // three CTAs per SM (shared memory)
        if (blocks > pp.n_units) blocks = pp.n_units;
        if (p.D == 128) launch_pdl(pool_kernel<128>, (unsigned)blocks, kPoolThreads, PoolCfg<128>::SMEM, st, tq, tk, p, pp);
        else launch_pdl(pool_kernel<64>, (unsigned)blocks, kPoolThreads, PoolCfg<64>::SMEM, st, tq, tk, p, pp);
        const dim3 sg(nblk(p.n_cand, kScoreTile) * nblk(p.n_qb, kScoreTile), (unsigned)p.H);
        launch_pdl(score_kernel, sg, 256, 0, st, p, (const float *)qmean, (const float *)kmean);
        const int npow2 = pow2_at_least(p.n_cand);
        const unsigned groups = (unsigned)(((p.n_qb + 1) / 2 + 3) / 4);
        if (p.keep <= 128 && p.n_cand <= 1024) launch_pdl(select_lists_top128_kernel, p.H * groups, 256, 0, st, p);
        else if (npow2 <= 256) launch_pdl(select_lists_warp_kernel<8>, p.H * groups, 256, 0, st, p);
        else if (npow2 <= 512) launch_pdl(select_lists_warp_kernel<16>, p.H * groups, 256, 0, st, p);
        else if (npow2 <= 1024) launch_pdl(select_lists_warp_kernel<32>, p.H * groups, 256, 0, st, p);
        else launch_pdl(select_lists_kernel, p.H * ((p.n_qb + 1) / 2), 256, select_smem(npow2, p.n_cand), st, p, npow2);
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
