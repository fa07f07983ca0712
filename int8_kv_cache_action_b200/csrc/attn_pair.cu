// attn_pair_kernel: the attention of nomas_attn_run at head_dim 128 with the two query blocks that share a
// tile list in one CTA (fluxbbs.com "架构" for the visibility; "单卡 4090 怎么做到的" for INT8 storage and
// the sparse mode).  The arithmetic is attn_fwd_kernel's (fp16 operands, fp32 accumulation, per-key
// scales in fp32, log2-domain softmax with the lazy rescale); what changes is the schedule.
//
// One CTA = one head x one pair of 128-row query blocks (query tiles 0 and 1).  Roles (12 warps, one CTA
// per SM):
//   warps 0-3   softmax of query tile 0: one thread per row, all 128 key columns of a tile
//   warps 4-7   softmax of query tile 1
//   warp 8      tcgen05.mma issuer (one thread) and TMEM owner
//   warp 9      TMA producer (one thread)
//   warps 10-11 column info: key scale, value scale and visibility code of every column, one entry
//               ahead, in a four-deep shared-memory ring (two columns per thread)
// Registers: launched at 168 per thread (384 x 168 = 64512); setmaxnreg moves them to 216 for each
// softmax warpgroup and 72 for the third: 2 x 216 + 72 = 504 = 3 x 168.
//
// TMEM (512 columns): S_0 [0, 128), S_1 [128, 256), O_0 [256, 384), O_1 [384, 512); P_t (fp16 pairs)
// overwrites the first 64 columns of S_t once the row's 128 scores are in registers.
// Shared memory: Q_0 and Q_1 (fp16, converted from bf16 by the softmax threads) and rings of two K and
// two V^T tiles, all 128-byte swizzled K-major; the column-info ring.
//
//   S_t = Q_t K_j^T     SS MMA (A = Q_t, B = K_j)
//   O_t += P_t V_j      TS MMA (A = P_t in TMEM, B = V_j^T)
//
// The list is walked once by every role; an entry is used by query tile t when it carries t's use bit.
// For each entry the issuer runs, per query tile: the PV of the previous entry (once that tile's P is
// stored), then the tile's S.  So the tensor pipe alternates between the tiles: while the softmax of
// tile 0 works on S_0(j), the pipe computes PV_1(j-1) and S_1(j), and the other way round.  Because
// PV_t(j-1) is issued before S_t(j), the completion of S_t(j) implies that of PV_t(j-1): the softmax
// may rescale O_t as soon as it sees S_t(j), and S_t(j) may overwrite P_t(j-1) (in-order execution).
// A tile skipped by one query tile costs that tile's warps only the column-info hand-off.
//
// Grid: one CTA per work unit (head, pair), head-major.  For a dense call whose units leave a partial
// last wave, the host splits each left-over unit into list shares (AttnParams::n_full / tail_*): such
// a CTA runs one share and writes unnormalised partials that attn_combine_tail_kernel merges.
#include <cmath>
#include <cuda_fp16.h>

#include "attn.cuh"
#include "common.cuh"

namespace nomas {

constexpr int kPairThreads = 384;
constexpr int kPairWarpMma = 8, kPairWarpTma = 9, kPairWarpCi = 10;   // column info: warps 10-11
constexpr int kPairRegSoftmax = 216, kPairRegOther = 72;
static_assert(2 * kPairRegSoftmax + kPairRegOther == 3 * 168, "register split must equal the launch total");
constexpr int kPairNCI = 4;                    // column-info ring depth
constexpr uint32_t kTmO = 256;                 // O_t at kTmO + 128 t; S_t at 128 t

struct PairCfg {
    static constexpr int D = 128;
    static constexpr int SLOT = kTile * D * 2;          // one fp16 tile (32 KB)
    static constexpr int PANEL = kTile * 128;           // 64 fp16 columns of 128 rows (16 KB)
    static constexpr int NK = 2, NV = 2;                // K and V^T slots
    static constexpr int OFF_Q = 0;                     // Q_0, Q_1
    static constexpr int OFF_K = OFF_Q + 2 * SLOT;
    static constexpr int OFF_V = OFF_K + NK * SLOT;
    static constexpr int OFF_CS = OFF_V + NV * SLOT;    // float [kPairNCI][128] key scale x log2 e
    static constexpr int OFF_CV = OFF_CS + kPairNCI * 512;    // float [kPairNCI][128] value scale
    static constexpr int OFF_CW = OFF_CV + kPairNCI * 512;    // int4  [kPairNCI][128] visibility codes
    static constexpr int OFF_BAR = OFF_CW + kPairNCI * 2048;
    // q_ready; k_full, k_empty [NK]; v_full, v_empty [NV]; ci_full, ci_empty [kPairNCI]; s_full, p_full [2];
    // o_final
    static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 2 * kPairNCI + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int SMEM = BYTES + 1024;           // slack for 1024-byte alignment
};
static_assert(PairCfg::SMEM <= 227 * 1024, "shared memory of the pair kernel");

__global__ void __launch_bounds__(kPairThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_kt,
                     const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_vt,
                     const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_kp,
                     const __grid_constant__ CUtensorMap tm_vh, const __grid_constant__ CUtensorMap tm_vp,
                     const AttnParams p) {
    using C = PairCfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t *sQ = sm + C::OFF_Q;
    uint8_t *sK = sm + C::OFF_K;
    uint8_t *sV = sm + C::OFF_V;
    float *sCS = reinterpret_cast<float *>(sm + C::OFF_CS);
    float *sCV = reinterpret_cast<float *>(sm + C::OFF_CV);
    int4 *sCW = reinterpret_cast<int4 *>(sm + C::OFF_CW);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *q_ready = bars;
    uint64_t *k_full = bars + 1, *k_empty = k_full + C::NK;
    uint64_t *v_full = k_empty + C::NK, *v_empty = v_full + C::NV;
    uint64_t *ci_full = v_empty + C::NV, *ci_empty = ci_full + kPairNCI;
    uint64_t *s_full = ci_empty + kPairNCI, *p_full = s_full + 2, *o_final = p_full + 2;
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // work unit (head-major: the CTAs of one head run close together and share its K / V^T in L2) and,
    // for a unit of the split tail, its share
    int unit = blockIdx.x, tshare = 0;
    const bool tail = p.tail_len > 0 && unit >= p.n_full;
    if (tail) {
        const int t = unit - p.n_full;
        unit = p.n_full + t / p.tail_shares;
        tshare = t - (t / p.tail_shares) * p.tail_shares;
    }
    const int h = unit / p.n_pairs;
    const int pair = unit - h * p.n_pairs;
    constexpr int kBoth = kUse0 | kUse1;
    const int list_id = p.sparse ? h * p.n_pairs + pair : pair;
    const int4 *list = p.lists + (int64_t)list_id * p.expect.list_cap;   // advanced to this CTA's share below

    // header check (every thread reads the same words; all take the same branch)
    const MaskHeader *hd = reinterpret_cast<const MaskHeader *>(p.mask);
    const bool hdr_ok = hd->magic == p.expect.magic && hd->mode == p.expect.mode &&
                        hd->n_qblocks == p.expect.n_qblocks && hd->n_lists == p.expect.n_lists &&
                        hd->history_tokens == p.expect.history_tokens && hd->head_tokens == p.expect.head_tokens &&
                        hd->cache_version == p.expect.cache_version && hd->n_query == p.expect.n_query &&
                        hd->text_tokens == p.expect.text_tokens && hd->list_cap == p.expect.list_cap;
    const WsHeader *wh = p.ws_hdr;
    const bool ws_ok = wh->magic == p.ws_expect.magic && wh->head_dim == p.ws_expect.head_dim &&
                       wh->cache_version == p.ws_expect.cache_version &&
                       wh->head_tokens == p.ws_expect.head_tokens &&
                       wh->history_tokens == p.ws_expect.history_tokens && wh->n_query == p.ws_expect.n_query &&
                       wh->text_tokens == p.ws_expect.text_tokens;
    if (!hdr_ok || !ws_ok) {
        if (threadIdx.x == 0) set_device_error(p.err, NOMAS_EDEVICE, hdr_ok ? 2 : 1);
        return;
    }
    // this CTA's share of the list (a share past the list's end has nothing to do: the merge skips it)
    const int n_all = p.counts[list_id];
    const bool partial = p.share_len > 0 || tail;
    const int slen = tail ? p.tail_len : p.share_len;
    const int lo = partial ? (tail ? tshare : (int)blockIdx.z) * slen : 0;
    if (partial && lo >= n_all) return;
    const int n_tiles = partial ? min(slen, n_all - lo) : n_all;
    list += lo;

    if (threadIdx.x == 0) {
        mbar_init(q_ready, 8);
        for (int i = 0; i < C::NK; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < C::NV; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < kPairNCI; ++i) {
            mbar_init(&ci_full[i], 2);      // the 2 column-info warps
            mbar_init(&ci_empty[i], 8);     // the 8 softmax warps, for every entry
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 4);       // the query tile's 4 softmax warps
        }
        mbar_init(o_final, 1);
        misc[1] = 0;
        fence_mbar_init();
    }
    if (warp == kPairWarpMma) {
        tmem_alloc(&misc[0], 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    Watchdog wd{p.err, abort_flag, p.timeout_ns, 0};

    if (warp >= kPairWarpMma) {
        setmaxnreg_dec<kPairRegOther>();
        if (warp >= kPairWarpCi) {
            // -------------------------------------------------------------- column info
            // Thread t writes columns t and t + 64 of every entry; each warp arrives on ci_full.
            wd.where = 3;
            const int t = threadIdx.x - 32 * kPairWarpCi;   // 0..63
            ListCursor cursor(list, n_tiles);
            int u = 0;
            int4 en;
            bool have = cursor.next(kBoth, en);
            ColInfo n0, n1;
            if (have) {
                const bool m = (en.x & (kMask0 | kMask1)) != 0;
                n0 = column_info(p, h, en, t, m);
                n1 = column_info(p, h, en, t + 64, m);
            }
            while (have) {
                const ColInfo c0 = n0, c1 = n1;
                have = cursor.next(kBoth, en);
                if (have) {
                    const bool m = (en.x & (kMask0 | kMask1)) != 0;
                    n0 = column_info(p, h, en, t, m);
                    n1 = column_info(p, h, en, t + 64, m);
                }
                const int ci = u % kPairNCI;
                if (!__all_sync(0xffffffffu, mbar_wait(&ci_empty[ci], ((u / kPairNCI) & 1) ^ 1, wd, 1))) break;
                sCS[ci * 128 + t] = p.scale_log2 * c0.ks;
                sCS[ci * 128 + t + 64] = p.scale_log2 * c1.ks;
                sCV[ci * 128 + t] = c0.vs;
                sCV[ci * 128 + t + 64] = c1.vs;
                if (c0.masked) {
                    sCW[ci * 128 + t] = make_int4(c0.w.x, c0.w.y, c0.w.z, c0.w.w);
                    sCW[ci * 128 + t + 64] = make_int4(c1.w.x, c1.w.y, c1.w.z, c1.w.w);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ci_full[ci]);
                ++u;
            }
        } else if (warp == kPairWarpMma && lane == 0) {
            // -------------------------------------------------------------- MMA issuer
            wd.where = 4;
            constexpr uint32_t idesc = idesc_f16_f32(128, 128, false, false);
            const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
            bool ok = mbar_wait(q_ready, 0, wd, 1);
            tc_fence_after();
            int cnt[2] = {0, 0};             // S MMAs issued per query tile (phases of p_full)
            bool pend[2] = {false, false};   // PV of the previous entry not yet issued
            bool acc_on[2] = {false, false}; // O_t holds a product
            // PV_t of entry `ent` once query tile t's P is stored and V^T has landed
            auto issue_pv = [&](int t, int ent) -> bool {
                // the P hand-off is on the critical path of each query tile: poll without suspending
                if (!mbar_wait_spin(&p_full[t], (cnt[t] - 1) & 1, wd, 3)) return false;
                const int sv = ent % C::NV;
                if (!mbar_wait(&v_full[sv], (ent / C::NV) & 1, wd, 4)) return false;
                tc_fence_after();
                const uint32_t vb = v_addr + sv * C::SLOT;
                const uint32_t tP = tmem + 128u * t, tO = tmem + kTmO + 128u * t;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tO, tP + kk * 8, sdesc_sw128(vb + (kk / 4) * C::PANEL + (kk % 4) * 32, 16, 1024), idesc,
                            (acc_on[t] || kk > 0) ? 1u : 0u);
                acc_on[t] = true;
                return true;
            };
            int u = 0;
            ListCursor cursor(list, n_tiles);
            int4 e;
            while (ok && cursor.next(kBoth, e)) {
                const int sk = u % C::NK;
                bool k_ready = false, any_pv = false;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!ok) break;
                    if (pend[t]) {
                        ok = issue_pv(t, u - 1);
                        pend[t] = false;
                        any_pv = true;
                        if (!ok) break;
                    }
                    if (e.x & (t ? kUse1 : kUse0)) {
                        if (!k_ready) {
                            ok = mbar_wait(&k_full[sk], (u / C::NK) & 1, wd, 2);
                            if (!ok) break;
                            tc_fence_after();
                            k_ready = true;
                        }
                        const uint32_t kb = k_addr + sk * C::SLOT, qa = q_addr + t * C::SLOT;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_ss(tmem + 128u * t, sdesc_sw128(qa + (kk / 4) * C::PANEL + (kk % 4) * 32, 16, 1024),
                                    sdesc_sw128(kb + (kk / 4) * C::PANEL + (kk % 4) * 32, 16, 1024), idesc,
                                    kk > 0 ? 1u : 0u);
                        umma_commit(&s_full[t]);
                        ++cnt[t];
                        pend[t] = true;
                    }
                }
                if (!ok) break;
                if (any_pv) umma_commit(&v_empty[(u - 1) % C::NV]);   // both PVs of entry u - 1 issued
                umma_commit(&k_empty[sk]);                            // every S of entry u issued
                ++u;
            }
            if (ok) {
                bool any_pv = false;
                for (int t = 0; t < 2 && ok; ++t)
                    if (pend[t]) {
                        ok = issue_pv(t, u - 1);
                        any_pv = true;
                    }
                if (ok && any_pv) umma_commit(&v_empty[(u - 1) % C::NV]);
            }
            umma_commit(o_final);
            // the MMAs must be complete before the CTA releases TMEM, also on the abort path
            if (!ok) mbar_drain(o_final, 0, 100000000ull);
        } else if (warp == kPairWarpTma && lane == 0) {
            // -------------------------------------------------------------- TMA producer
            wd.where = 5;
            prefetch_tmap(&tm_kc);
            prefetch_tmap(&tm_vc);
            prefetch_tmap(&tm_kh);
            prefetch_tmap(&tm_vh);
            uint32_t kpend = 0, vpend = 0;           // per slot: a copy was issued
            uint32_t kwpar = 0, vwpar = 0;           // per slot: parity of the phase it completes
            int u = 0;
            ListCursor cursor(list, n_tiles);
            int4 e;
            while (cursor.next(kBoth, e)) {
                const int kind = e.x & 3;
                const int start = e.y;
                const CUtensorMap *mk = kind == kKindCur ? &tm_kc : kind == kKindText ? &tm_kt
                                      : kind == kKindHist ? &tm_kh : &tm_kp;
                const CUtensorMap *mv = kind == kKindCur ? &tm_vc : kind == kKindText ? &tm_vt
                                      : kind == kKindHist ? &tm_vh : &tm_vp;
                const int sk = u % C::NK;
                if (!mbar_wait(&k_empty[sk], ((u / C::NK) & 1) ^ 1, wd, 1)) break;
                uint8_t *dk = sK + sk * C::SLOT;
                mbar_arrive_expect_tx(&k_full[sk], C::SLOT);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) tma_load_3d(dk + hh * C::PANEL, mk, &k_full[sk], hh * 64, start, h);
                kpend |= 1u << sk;
                kwpar = (kwpar & ~(1u << sk)) | ((uint32_t)((u / C::NK) & 1) << sk);
                const int sv = u % C::NV;
                if (!mbar_wait(&v_empty[sv], ((u / C::NV) & 1) ^ 1, wd, 2)) break;
                uint8_t *dv = sV + sv * C::SLOT;
                mbar_arrive_expect_tx(&v_full[sv], C::SLOT);
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) tma_load_3d(dv + pp * C::PANEL, mv, &v_full[sv], start + 64 * pp, 0, h);
                vpend |= 1u << sv;
                vwpar = (vwpar & ~(1u << sv)) | ((uint32_t)((u / C::NV) & 1) << sv);
                ++u;
            }
            // the bulk copies must land before the CTA's shared memory is released (a no-op unless
            // this CTA is aborting)
            for (int i = 0; i < C::NK; ++i)
                if ((kpend >> i) & 1u) mbar_drain(&k_full[i], (kwpar >> i) & 1u, 100000000ull);
            for (int i = 0; i < C::NV; ++i)
                if ((vpend >> i) & 1u) mbar_drain(&v_full[i], (vwpar >> i) & 1u, 100000000ull);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax warpgroups
        // Waits are made warp-uniform (__all_sync) because tcgen05.ld/st are warp-collective.
        setmaxnreg_inc<kPairRegSoftmax>();
        const int qt = warp >> 2;           // query tile
        const int g = warp & 3;             // TMEM lane group
        wd.where = 1 + qt;
        const int r = g * 32 + lane;
        const int64_t row = ((int64_t)2 * pair + qt) * kTile + r;
        const bool row_ok = row < p.Nq;
        const int use_bit = qt ? kUse1 : kUse0, mask_bit = qt ? kMask1 : kMask0;
        // the row's visibility code, needed only on masked tiles and so rebuilt there
        auto row_code = [&]() -> VisCode {
            if (!p.text_rows) return row_video((int)fdiv(row_ok ? (uint32_t)row : 0u, p.divT));
            if (!row_ok || row < p.head_len) return row_head();
            const int2 w = p.txtwin[row];
            return row_tail(w.x, w.y);
        };
        // Q row -> fp16 -> this tile's 128-byte-swizzled rows (two 64-column panels)
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q + (row_ok ? row : 0) * p.tok_stride +
                                                               (int64_t)h * p.head_stride);
            uint8_t *qtile = sQ + qt * C::SLOT;
            bool bad = false;
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                const uint4 v = row_ok ? bf16x8_to_f16(__ldg(src + i)) : make_uint4(0, 0, 0, 0);
                bad |= f16x8_nonfinite(v);
                *reinterpret_cast<uint4 *>(qtile + (i / 8) * C::PANEL + sw128_offset((uint32_t)r, (uint32_t)(i % 8))) = v;
            }
            if (bad) set_device_error(p.err, NOMAS_ERANGE, 33);   // q outside the fp16 range
            fence_proxy_async_smem();                              // visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }
        const uint32_t lane_base = (uint32_t)(g * 32) << 16;
        const uint32_t tS = tmem + lane_base + 128u * qt;
        const uint32_t tO = tmem + lane_base + kTmO + 128u * qt;
        float m_used = -INFINITY;
        float l = 0.0f;
        int u = 0, j = 0;                   // entry index; tiles of this query tile
        bool ok = true;
        ListCursor cursor(list, n_tiles);
        int4 e;
        while (cursor.next(kBoth, e)) {
            const int ci = u % kPairNCI;
            ok = __all_sync(0xffffffffu, mbar_wait(&ci_full[ci], (u / kPairNCI) & 1, wd, 1));
            if (!ok) break;
            if (!(e.x & use_bit)) {         // the other query tile's entry: release the column info
                __syncwarp();
                if (lane == 0) mbar_arrive(&ci_empty[ci]);
                ++u;
                continue;
            }
            const bool masked = (e.x & mask_bit) != 0;
            const bool cached = is_cached(e.x & 3);
            // visibility of the 128 keys to the row, taken before the scores are loaded
            uint32_t vm[4] = {~0u, ~0u, ~0u, ~0u};
            if (masked) {
                const VisCode rc = row_code();
                const int4 *cw = sCW + ci * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t bits = 0;
#pragma unroll 8
                    for (int i = 0; i < 32; ++i) {
                        const int4 w = cw[q4 * 32 + i];
                        bits |= (visible(VisCode{w.x, w.y, w.z, w.w}, rc) ? 1u : 0u) << i;
                    }
                    vm[q4] = bits;
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[qt], j & 1, wd, 2));
            if (!ok) break;
            tc_fence_after();
            float s[128];
            tmem_ld128f_sync(tS, s);
            // cached keys: apply the per-key scale (which carries softmax scale * log2 e) to the score
            if (cached) {
                const float4 *cs4 = reinterpret_cast<const float4 *>(sCS + ci * 128);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if ((i & 7) == 0) asm volatile("" ::: "memory");   // bound how far loads are hoisted
                    const float4 v = cs4[i];
                    const float2 a = __fmul2_rn(make_float2(s[4 * i], s[4 * i + 1]), make_float2(v.x, v.y));
                    const float2 c = __fmul2_rn(make_float2(s[4 * i + 2], s[4 * i + 3]), make_float2(v.z, v.w));
                    s[4 * i] = a.x;
                    s[4 * i + 1] = a.y;
                    s[4 * i + 2] = c.x;
                    s[4 * i + 3] = c.y;
                }
            }
            if (masked) {
#pragma unroll
                for (int i = 0; i < 128; ++i) s[i] = ((vm[i >> 5] >> (i & 31)) & 1u) ? s[i] : -INFINITY;
            }
            // row maximum: four independent max3 chains of 32 columns
            float mc[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float m = max3(s[32 * k], s[32 * k + 1], s[32 * k + 2]);
#pragma unroll
                for (int c = 3; c < 31; c += 2) m = max3(m, s[32 * k + c], s[32 * k + c + 1]);
                mc[k] = fmaxf(m, s[32 * k + 31]);
            }
            const float pm = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
            // log2 domain: cached scores are already scaled, bf16-source scores take the uniform scale
            // (a positive factor commutes with the maximum exactly)
            const float cmul = cached ? 1.0f : p.scale_log2;
            const float mt = pm * cmul;
            const float m_new = fmaxf(m_used, mt);
            const bool grow = m_new > m_used + kRescaleThreshold;   // false while both are -inf
            const bool need_o = grow && m_used != -INFINITY;
            const float f = need_o ? ex2(m_used - m_new) : 1.0f;
            if (grow) m_used = m_new;
            const float off = (m_used == -INFINITY) ? 0.0f : m_used;
            const float2 cm2 = make_float2(cmul, cmul);
            const float2 no2 = make_float2(-off, -off);
            float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
            const float2 *cv2 = reinterpret_cast<const float2 *>(sCV + ci * 128);
#pragma unroll
            for (int qc = 0; qc < 4; ++qc) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 a = __ffma2_rn(make_float2(s[qc * 32 + c], s[qc * 32 + c + 1]), cm2, no2);
                    float2 pe = (c / 2) < kPolyPairs ? exp2_poly(a) : make_float2(ex2(a.x), ex2(a.y));
                    acc[(c >> 1) & 1] = __fadd2_rn(acc[(c >> 1) & 1], pe);
                    // cached values enter the tensor core as exact codes: P carries their scale
                    if (cached) pe = __fmul2_rn(pe, cv2[(qc * 32 + c) / 2]);
                    pk[c / 2] = f16x2_of(pe.x, pe.y);
                }
                tmem_st16(tS + qc * 16, pk);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ci_empty[ci]);   // column info no longer needed
            l = l * f + ((acc[0].x + acc[1].x) + (acc[0].y + acc[1].y));
            // rescale O_t (rare: only when some row's maximum grew past the threshold); S_t(j)'s
            // completion implies PV_t(j-1)'s, and PV_t(j) waits for the P hand-off below
            if (__any_sync(0xffffffffu, need_o)) {
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t rr[32];
                    tmem_ld32_sync(tO + c0, rr);
#pragma unroll
                    for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
                    tmem_st32(tO + c0, rr);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[qt]);
            ++j;
            ++u;
        }
        // epilogue: O / l
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_final, 0, wd, 5));
        if (ok) {
            tc_fence_after();
            const float inv = partial ? 1.0f : (l > 0.0f ? 1.0f / l : 0.0f);
            const int64_t trow = ((int64_t)tshare * p.n_tail + (unit - p.n_full)) * (2 * kTile) + qt * kTile + r;
            float *dst = tail      ? p.tail_o + trow * D
                         : partial ? p.part_o + ((int64_t)blockIdx.z * p.Nq * p.H + row * p.H + h) * D
                                   : p.out + (row * p.H + h) * (int64_t)D;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t rr[32];
                tmem_ld32_sync(tO + c0, rr);
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 v = make_float4(__uint_as_float(rr[i]) * inv, __uint_as_float(rr[i + 1]) * inv,
                                               __uint_as_float(rr[i + 2]) * inv, __uint_as_float(rr[i + 3]) * inv);
                        if (l == 0.0f) v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);   // no visible key (in this share)
                        *reinterpret_cast<float4 *>(dst + c0 + i) = v;
                    }
                }
            }
            if (tail && row_ok)
                p.tail_ml[trow] = make_float2(m_used, l);
            else if (partial && row_ok)
                p.part_ml[((int64_t)blockIdx.z * p.H + h) * p.Nq + row] = make_float2(m_used, l);
            else if (p.lse && row_ok)
                p.lse[(int64_t)h * p.Nq + row] = (m_used + log2f(l)) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kPairWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Merge of the split tail of a dense pair-kernel call: one warp per (tail unit, row of its query-block
// pair); the unit's list of the block pair gives how many shares ran.
template <int D>
__global__ void __launch_bounds__(256) attn_combine_tail_kernel(const AttnParams p) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (int64_t)p.n_tail * 2 * kTile) return;          // warp-uniform
    const int tu = (int)(w / (2 * kTile)), rr = (int)(w - (int64_t)tu * 2 * kTile);
    const int unit = p.n_full + tu;
    const int h = unit / p.n_pairs, pair = unit - h * p.n_pairs;
    const int64_t row = (int64_t)pair * 2 * kTile + rr;
    if (row >= p.Nq) return;
    const int n_share = min(p.tail_shares, (p.counts[pair] + p.tail_len - 1) / p.tail_len);
    const int64_t t0 = (int64_t)tu * 2 * kTile + rr, stride = (int64_t)p.n_tail * 2 * kTile;
    merge_shares<D>(p.tail_o + t0 * D, stride * D, p.tail_ml + t0, stride, n_share, p.out + (row * p.H + h) * (int64_t)D,
                    p.lse ? p.lse + (int64_t)h * p.Nq + row : nullptr, lane);
}

int launch_combine_tail(const AttnParams &p, int D, cudaStream_t st) {
    if (D != 128) return NOMAS_EUNSUPPORTED;
    const int64_t warps = (int64_t)p.n_tail * 2 * kTile;
    attn_combine_tail_kernel<128><<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(p);
    return check_launch("attn_combine_tail_kernel launch");
}

int launch_attn_pair(const AttnParams &p, dim3 grid, const CUtensorMap *maps, cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e =
            cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::SMEM);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(attn pair smem)", (int)e, cudaGetErrorString(e));
        attr_set = true;
    }
    attn_pair_kernel<<<grid, kPairThreads, PairCfg::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5],
                                                               maps[6], maps[7], p);
    return check_launch("attn_pair_kernel launch");
}

}  // namespace nomas
