// nomas_attn_fwd: action-aware segment-causal attention over an INT8 history (fluxbbs.com "架构" for
// the visibility; "单卡 4090 怎么做到的" for INT8 storage and the sparse mode).
//
// One CTA = one head x one 128-row query block.  Roles (16 warps, one CTA per SM):
//   warps 0-3   softmax over key columns 0-63 of every S tile (TMEM lanes 0-127, one thread per row)
//   warps 4-7   softmax over key columns 64-127; the two halves of a row swap their maxima through
//               shared memory, so both apply the same offset
//   warps 8-11  column info: per-column key scale, value scale and visibility code of every tile,
//               one tile ahead, in a four-deep shared-memory ring
//   warp 12     tcgen05.mma issuer (one thread) and TMEM owner
//   warp 13     TMA producer (one thread); warps 14-15 idle
// The register file is split per SM sub-partition (one warp of each warpgroup on each), so the
// kernel launches at 128 registers per thread and moves them with setmaxnreg: softmax 168 each,
// column info 112, MMA / producer warpgroup 64 -- 2*168 + 112 + 64 = 512 = 4 x 128.
//
// TMEM (512 columns): Q (fp16 pairs) at [0, D/2), S double buffer at [128, 256) and [256, 384),
// O at [384, 384 + D).  P (fp16) overwrites the first 32 columns of each 64-column half of its S
// buffer, so each softmax half writes only columns it has already read.
//
// Both products are TS MMAs (A from TMEM) with a K-major B in 128-byte-swizzled shared memory:
//   S_b  = Q K_j^T     B = K_j    [128 keys][D]
//   O   += P_j V_j     B = V_j^T  [D][128 keys]   (values are stored transposed by the pre-pass)
// For D = 128 the two share one instruction descriptor: a change of MMA shape between consecutive
// tcgen05.mma batches stalls the tensor pipe, and the pipe only reaches full rate with more than
// two batches in flight, which the S -> softmax -> PV dependency does not allow.  The issue order
// S_0, S_1, PV_0, S_2, PV_1, ... computes S_{j+1} while the softmax works on S_j; S_{j+2} reuses
// the buffer of S_j after PV_j, which tcgen05's in-order execution makes safe.
//
// Every tile reaches shared memory by TMA alone.  The pre-pass writes the operands in the layouts
// the boxes read: fp16 keys [H][n][D] and transposed fp16 values [H][D][n] for the current segment
// and the text (converted from bf16), and for the retained history and the description heads the
// INT8 codes as exact fp16 integers in the same layouts (-127..127 are exact in fp16), with their
// scales in age order.  Converting the codes once per call in the pre-pass costs one HBM pass over
// the history; converting them in shared memory inside this kernel took issue slots from the
// softmax warps on every history tile of every query block.
//
// Precision: every MMA operand is fp16 with fp32 accumulation.  bf16 inputs convert to fp16
// exactly for magnitudes in [2^-14, 65504] (the supported input range; smaller values keep 2^-24
// absolute resolution).  INT8 codes enter the tensor core exactly: a key's scale multiplies its fp32
// score, a value's scale multiplies the fp32 probability before P is rounded to fp16 (so P * v uses
// the product p * scale * code, rounded once).  Softmax uses a lazy rescale: the running offset
// moves only when the row maximum grows by more than 6 (log2 units), so p <= 64 and p * scale stays
// inside fp16 for every input in the supported range (absmax <= 65504 gives scale <= 516); O is
// then rescaled in TMEM once the previous PV has completed.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cuda_fp16.h>

#include "attn.cuh"
#include "common.cuh"
#include "prep.cuh"

namespace nomas {

constexpr int kAttnThreads = 512;
constexpr int kWarpCi = 8, kWarpMma = 12, kWarpTma = 13;  // column info: warps 8-11
constexpr int kRegSoftmax = 168, kRegLoader = 112, kRegMma = 64;
static_assert(2 * kRegSoftmax + kRegLoader + kRegMma == 4 * 128, "register split must equal the launch total");
constexpr int kNCI = 4;                     // column-info ring depth
constexpr uint32_t kTmQ = 0, kTmS = 128, kTmO = 384;

template <int D>
struct AttnCfg {
    static constexpr int NK = (D == 128) ? 3 : 6;          // K tile slots
    static constexpr int NV = NK;                          // V^T tile slots
    static constexpr int SLOT = kTile * D * 2;             // one fp16 tile
    static constexpr int KPANEL = kTile * 128;             // K: 64 columns (128 B) of 128 rows
    static constexpr int VPANEL = D * 128;                 // V^T: 64 keys (128 B) of D rows
    static constexpr int KSTEPS = D / 16;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + NK * SLOT;
    static constexpr int OFF_CS = OFF_V + NV * SLOT;       // float [kNCI][128] key scale x log2 e
    static constexpr int OFF_CV = OFF_CS + kNCI * 512;     // float [kNCI][128] value scale
    static constexpr int OFF_CW = OFF_CV + kNCI * 512;     // int4  [kNCI][128] key visibility codes
    static constexpr int OFF_XM = OFF_CW + kNCI * 2048;    // float [2 buffers][2 halves][128] maxima
    static constexpr int OFF_XL = OFF_XM + 2048;           // float [2 halves][128] row sums
    static constexpr int OFF_BAR = OFF_XL + 1024;
    // q_ready; k_full, k_empty [NK]; v_full, v_empty [NV]; ci_full, ci_empty [kNCI];
    // s_full, p_full, xm_bar [2]; pv_done; o_final; xl_bar
    static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 2 * kNCI + 6 + 3;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int SMEM = BYTES + 1024;              // slack for 1024-byte alignment
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_kt,
                    const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_vt,
                    const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_kp,
                    const __grid_constant__ CUtensorMap tm_vh, const __grid_constant__ CUtensorMap tm_vp,
                    const AttnParams p) {
    using C = AttnCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t *sK = sm + C::OFF_K;
    uint8_t *sV = sm + C::OFF_V;
    float *sCS = reinterpret_cast<float *>(sm + C::OFF_CS);
    float *sCV = reinterpret_cast<float *>(sm + C::OFF_CV);
    int4 *sCW = reinterpret_cast<int4 *>(sm + C::OFF_CW);
    float *sXM = reinterpret_cast<float *>(sm + C::OFF_XM);
    float *sXL = reinterpret_cast<float *>(sm + C::OFF_XL);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *q_ready = bars;
    uint64_t *k_full = bars + 1, *k_empty = k_full + C::NK;
    uint64_t *v_full = k_empty + C::NK, *v_empty = v_full + C::NV;
    uint64_t *ci_full = v_empty + C::NV, *ci_empty = ci_full + kNCI;
    uint64_t *s_full = ci_empty + kNCI, *p_full = s_full + 2, *xm_bar = p_full + 2;
    uint64_t *pv_done = xm_bar + 2, *o_final = pv_done + 1, *xl_bar = o_final + 1;
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qb = blockIdx.x;   // 128-row query block
    const int h = blockIdx.y;
    const int use_bit = (qb & 1) ? kUse1 : kUse0;
    const int mask_bit = (qb & 1) ? kMask1 : kMask0;
    const int list_id = p.sparse ? h * p.n_pairs + (qb >> 1) : (qb >> 1);
    const int4 *list = p.lists + (int64_t)list_id * p.expect.list_cap;   // advanced to this split's share below

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
    const bool partial = p.share_len > 0;
    const int lo = partial ? (int)blockIdx.z * p.share_len : 0;
    if (partial && lo >= n_all) return;
    const int n_tiles = partial ? min(p.share_len, n_all - lo) : n_all;
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
        for (int i = 0; i < kNCI; ++i) {
            mbar_init(&ci_full[i], 4);      // the 4 column-info warps
            mbar_init(&ci_empty[i], 8);     // the 8 softmax warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 8);
            mbar_init(&xm_bar[b], 8);
        }
        mbar_init(pv_done, 1);
        mbar_init(o_final, 1);
        mbar_init(xl_bar, 8);
        misc[1] = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&misc[0], 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    Watchdog wd{p.err, abort_flag, p.timeout_ns, 0};
    const int64_t qrow0 = (int64_t)qb * kTile;

    if (warp >= kWarpCi && warp < kWarpCi + 4) {
        // ------------------------------------------------------------------ column-info warpgroup
        // Thread t writes column t of every tile's entry in the ring; each warp arrives on ci_full for
        // its 32 columns.
        setmaxnreg_dec<kRegLoader>();
        wd.where = 3;
        const int t = threadIdx.x - 32 * kWarpCi;   // 0..127
        ListCursor cursor(list, n_tiles);
        int u = 0;                          // index among this block's tiles
        int4 en;
        bool have = cursor.next(use_bit, en);
        ColInfo nxt0;
        if (have) nxt0 = column_info(p, h, en, t, (en.x & mask_bit) != 0);
        while (have) {
            const ColInfo c0 = nxt0;
            have = cursor.next(use_bit, en);
            if (have) nxt0 = column_info(p, h, en, t, (en.x & mask_bit) != 0);
            const int ci = u % kNCI;
            if (!__all_sync(0xffffffffu, mbar_wait(&ci_empty[ci], ((u / kNCI) & 1) ^ 1, wd, 1))) break;
            sCS[ci * 128 + t] = p.scale_log2 * c0.ks;
            sCV[ci * 128 + t] = c0.vs;
            if (c0.masked) sCW[ci * 128 + t] = make_int4(c0.w.x, c0.w.y, c0.w.z, c0.w.w);
            __syncwarp();
            if (lane == 0) mbar_arrive(&ci_full[ci]);
            ++u;
        }
    } else if (warp >= kWarpMma) {
        setmaxnreg_dec<kRegMma>();
        if (warp == kWarpMma && lane == 0) {
            // -------------------------------------------------------------- MMA issuer
            wd.where = 4;
            constexpr uint32_t idesc_s = idesc_f16_f32(128, 128, false, false);
            constexpr uint32_t idesc_o = idesc_f16_f32(128, D, false, false);
            const uint32_t tQ = tmem + kTmQ, tO = tmem + kTmO;
            const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
            bool ok = mbar_wait(q_ready, 0, wd, 1);
            auto issue_pv = [&](int v) -> bool {
                const int sv = v % C::NV;
                if (!mbar_wait(&p_full[v & 1], (v >> 1) & 1, wd, 3)) return false;
                if (!mbar_wait(&v_full[sv], (v / C::NV) & 1, wd, 4)) return false;
                tc_fence_after();
                const uint32_t vb = v_addr + sv * C::SLOT;
                const uint32_t tP = tmem + kTmS + (v & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tO, tP + (kk / 4) * 64 + (kk % 4) * 8,
                            sdesc_sw128(vb + (kk / 4) * C::VPANEL + (kk % 4) * 32, 16, 1024), idesc_o,
                            (v > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&v_empty[sv]);
                umma_commit(pv_done);
                return true;
            };
            int u = 0;
            ListCursor cursor(list, n_tiles);
            int4 e;
            while (ok && cursor.next(use_bit, e)) {
                const int sk = u % C::NK;
                ok = mbar_wait(&k_full[sk], (u / C::NK) & 1, wd, 2);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kb = k_addr + sk * C::SLOT;
                const uint32_t tS = tmem + kTmS + (u & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS; ++kk)
                    umma_ts(tS, tQ + kk * 8, sdesc_sw128(kb + (kk / 4) * C::KPANEL + (kk % 4) * 32, 16, 1024),
                            idesc_s, kk > 0 ? 1u : 0u);
                umma_commit(&s_full[u & 1]);
                umma_commit(&k_empty[sk]);
                if (u >= 1) ok = issue_pv(u - 1);
                ++u;
            }
            if (ok && u >= 1) ok = issue_pv(u - 1);
            umma_commit(o_final);
            // the MMAs must be complete before the CTA releases TMEM, also on the abort path
            if (!ok) mbar_drain(o_final, 0, 100000000ull);
        } else if (warp == kWarpTma && lane == 0) {
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
            while (cursor.next(use_bit, e)) {
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
                for (int hh = 0; hh < D / 64; ++hh) tma_load_3d(dk + hh * C::KPANEL, mk, &k_full[sk], hh * 64, start, h);
                kpend |= 1u << sk;
                kwpar = (kwpar & ~(1u << sk)) | ((uint32_t)((u / C::NK) & 1) << sk);
                const int sv = u % C::NV;
                if (!mbar_wait(&v_empty[sv], ((u / C::NV) & 1) ^ 1, wd, 2)) break;
                uint8_t *dv = sV + sv * C::SLOT;
                mbar_arrive_expect_tx(&v_full[sv], C::SLOT);
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) tma_load_3d(dv + pp * C::VPANEL, mv, &v_full[sv], start + 64 * pp, 0, h);
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
        setmaxnreg_inc<kRegSoftmax>();
        const int half = warp >> 2;         // key columns [64 * half, 64 * half + 64) of each tile
        const int g = warp & 3;             // TMEM lane group
        wd.where = 1 + half;
        const int r = g * 32 + lane;
        const int64_t row = qrow0 + r;
        const bool row_ok = row < p.Nq;
        // the row's visibility code (a video frame, or a text row of the head or of a tail), needed only
        // on masked tiles and so rebuilt there instead of held in registers
        auto row_code = [&]() -> VisCode {
            if (!p.text_rows) return row_video((int)fdiv(row_ok ? (uint32_t)row : 0u, p.divT));
            if (!row_ok || row < p.head_len) return row_head();
            const int2 w = p.txtwin[row];
            return row_tail(w.x, w.y);
        };
        const uint32_t lane_base = (uint32_t)(g * 32) << 16;
        constexpr int DH = D / 2;           // head-dim elements of Q and O handled by this half
        // Q row r, elements [half * DH, half * DH + DH) -> fp16 pairs in TMEM
        {
            uint32_t qp[DH / 2];
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q + (row_ok ? row : 0) * p.tok_stride +
                                                               (int64_t)h * p.head_stride + half * DH);
            bool bad = false;
#pragma unroll
            for (int i = 0; i < DH / 8; ++i) {
                const uint4 v = row_ok ? bf16x8_to_f16(__ldg(src + i)) : make_uint4(0, 0, 0, 0);
                bad |= f16x8_nonfinite(v);
                qp[4 * i] = v.x;
                qp[4 * i + 1] = v.y;
                qp[4 * i + 2] = v.z;
                qp[4 * i + 3] = v.w;
            }
            if (bad) set_device_error(p.err, NOMAS_ERANGE, 33);   // q outside the fp16 range
            const uint32_t tq = tmem + lane_base + kTmQ + (uint32_t)(half * DH / 2);
            if constexpr (DH / 2 == 32) {
                tmem_st32(tq, qp);
            } else {
                tmem_st16(tq, qp);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }
        float m_used = -INFINITY;
        float l = 0.0f;
        int u = 0;
        bool ok = true;
        ListCursor cursor(list, n_tiles);
        int4 e;
        while (cursor.next(use_bit, e)) {
            const int ci = u % kNCI;
            const int b = u & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&ci_full[ci], (u / kNCI) & 1, wd, 1));
            if (!ok) break;
            const bool masked = (e.x & mask_bit) != 0;
            const bool cached = is_cached(e.x & 3);
            // visibility of this half's 64 keys to the row, taken before the scores are loaded
            uint32_t vm[2] = {~0u, ~0u};
            if (masked) {
                const VisCode rc = row_code();
                const int4 *cw = sCW + ci * 128 + half * 64;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t bits = 0;
#pragma unroll 8
                    for (int i = 0; i < 32; ++i) {
                        const int4 w = cw[q2 * 32 + i];
                        bits |= (visible(VisCode{w.x, w.y, w.z, w.w}, rc) ? 1u : 0u) << i;
                    }
                    vm[q2] = bits;
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (u >> 1) & 1, wd, 2));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + lane_base + kTmS + (uint32_t)(b * 128 + half * 64);
            float s[64];
            tmem_ld64f_sync(tS, s);
            // cached keys: apply the per-key scale (which carries softmax scale * log2 e) to the score
            if (cached) {
                const float4 *cs4 = reinterpret_cast<const float4 *>(sCS + ci * 128 + half * 64);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
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
                for (int i = 0; i < 64; ++i) s[i] = ((vm[i >> 5] >> (i & 31)) & 1u) ? s[i] : -INFINITY;
            }
            // row maximum over this half (two independent max3 chains), then swapped with the other half
            float m0 = max3(s[0], s[1], s[2]), m1 = max3(s[32], s[33], s[34]);
#pragma unroll
            for (int c = 3; c < 31; c += 2) {
                m0 = max3(m0, s[c], s[c + 1]);
                m1 = max3(m1, s[32 + c], s[33 + c]);
            }
            const float pm = fmaxf(fmaxf(m0, s[31]), fmaxf(m1, s[63]));
            sXM[(b * 2 + half) * 128 + r] = pm;
            __syncwarp();
            if (lane == 0) mbar_arrive(&xm_bar[b]);
            ok = __all_sync(0xffffffffu, mbar_wait(&xm_bar[b], (u >> 1) & 1, wd, 3));
            if (!ok) break;
            const float po = sXM[(b * 2 + (half ^ 1)) * 128 + r];
            // log2 domain: cached scores are already scaled, bf16-source scores take the uniform scale
            // (a positive factor commutes with the maximum exactly); both halves compute the same values
            const float cmul = cached ? 1.0f : p.scale_log2;
            const float mt = fmaxf(pm, po) * cmul;
            const float m_new = fmaxf(m_used, mt);
            const bool grow = m_new > m_used + kRescaleThreshold;   // false while both are -inf
            const bool need_o = grow && m_used != -INFINITY;
            const float f = need_o ? ex2(m_used - m_new) : 1.0f;
            if (grow) m_used = m_new;
            const float off = (m_used == -INFINITY) ? 0.0f : m_used;
            const float2 cm2 = make_float2(cmul, cmul);
            const float2 no2 = make_float2(-off, -off);
            float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
            const float2 *cv2 = reinterpret_cast<const float2 *>(sCV + ci * 128 + half * 64);
#pragma unroll
            for (int qt = 0; qt < 2; ++qt) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 a = __ffma2_rn(make_float2(s[qt * 32 + c], s[qt * 32 + c + 1]), cm2, no2);
                    float2 pe = (c / 2) < kPolyPairs ? exp2_poly(a) : make_float2(ex2(a.x), ex2(a.y));
                    acc[(c >> 1) & 1] = __fadd2_rn(acc[(c >> 1) & 1], pe);
                    // cached values enter the tensor core as exact codes: P carries their scale
                    if (cached) pe = __fmul2_rn(pe, cv2[(qt * 32 + c) / 2]);
                    pk[c / 2] = f16x2_of(pe.x, pe.y);
                }
                tmem_st16(tS + qt * 16, pk);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ci_empty[ci]);   // column info no longer needed
            l = l * f + ((acc[0].x + acc[1].x) + (acc[0].y + acc[1].y));
            // rescale this half of O (rare: only when some row's maximum grew past the threshold) once
            // PV of the previous tile is complete; S_u's completion already implies PV_{u-2}'s
            if (__any_sync(0xffffffffu, need_o)) {
                ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (u - 1) & 1, wd, 4));
                if (!ok) break;
                tc_fence_after();
                const uint32_t tO = tmem + lane_base + kTmO + (uint32_t)(half * DH);
#pragma unroll 1
                for (int c0 = 0; c0 < DH; c0 += 32) {
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
            if (lane == 0) mbar_arrive(&p_full[b]);
            ++u;
        }
        // epilogue: the two halves' row sums, then O / l over this half's columns
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_final, 0, wd, 5));
        if (ok) {
            sXL[half * 128 + r] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(xl_bar);
            ok = __all_sync(0xffffffffu, mbar_wait(xl_bar, 0, wd, 6));
        }
        if (ok) {
            tc_fence_after();
            const float lt = l + sXL[(half ^ 1) * 128 + r];
            const float inv = partial ? 1.0f : (lt > 0.0f ? 1.0f / lt : 0.0f);
            float *dst = (partial ? p.part_o + (int64_t)blockIdx.z * p.Nq * p.H * D : p.out) +
                         (row * p.H + h) * (int64_t)D + half * DH;
            const uint32_t tO = tmem + lane_base + kTmO + (uint32_t)(half * DH);
#pragma unroll 1
            for (int c0 = 0; c0 < DH; c0 += 32) {
                uint32_t rr[32];
                tmem_ld32_sync(tO + c0, rr);
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 v = make_float4(__uint_as_float(rr[i]) * inv, __uint_as_float(rr[i + 1]) * inv,
                                               __uint_as_float(rr[i + 2]) * inv, __uint_as_float(rr[i + 3]) * inv);
                        if (lt == 0.0f) v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);   // no visible key (in this share)
                        *reinterpret_cast<float4 *>(dst + c0 + i) = v;
                    }
                }
            }
            if (partial && row_ok && half == 0)
                p.part_ml[((int64_t)blockIdx.z * p.H + h) * p.Nq + row] = make_float2(m_used, lt);
            else if (p.lse && row_ok && half == 0)
                p.lse[(int64_t)h * p.Nq + row] = (m_used + log2f(lt)) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace nomas

// Merge of the list shares of a text-row call: per (row, head), over the shares that saw a visible key,
// with M the largest offset, O = sum_s O_s 2^(m_s - M) / sum_s l_s 2^(m_s - M) and lse = (M + log2 of
// the denominator) ln 2 (the kernel's log2 domain).  Shares past the end of the row's list were not
// run and are not read.  One warp per (row, head), D / 32 channels per lane.
namespace nomas {
template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const float *part_o, const float2 *part_ml,
                                                           const int32_t *counts, int share_len, int64_t Nq,
                                                           int H, float *out, float *lse) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= Nq * H) return;                       // warp-uniform
    const int64_t row = w / H;
    const int h = (int)(w - row * H);
    const int n_share = (counts[row >> 8] + share_len - 1) / share_len;   // list of the block pair
    merge_shares<D>(part_o + (row * H + h) * (int64_t)D, Nq * H * (int64_t)D, part_ml + (int64_t)h * Nq + row,
                    (int64_t)H * Nq, n_share, out + (row * H + h) * (int64_t)D, lse ? lse + (int64_t)h * Nq + row : nullptr,
                    lane);
}
}  // namespace nomas

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
namespace nomas {

// 3-D tiled map.  dims / strides are innermost first (strides in bytes for dims 1 and 2).
static bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, const cuuint64_t dims[3],
                     const cuuint64_t strides[2], const cuuint32_t box[3], CUtensorMapSwizzle swz) {
    return make_tensor_map_3d(m, dt, base, dims, strides, box, swz);
}

static int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Workspace regions (256-byte aligned) after a 256-byte header, sized for the largest history the
// cache can retain so that the size does not depend on the cache state:
//   kc, kt   fp16 [H][n][D]       current-segment / text keys
//   vc, vt   fp16 [H][D][np8]     current-segment / text values, transposed
//   kh       fp16 [H][Lh][D]      retained-history key codes in age order
//   vht      fp16 [H][D][lhp]     retained-history value codes, transposed
//   ksl, vsl fp32 [H][lhp]        their scales
//   kp       fp16 [H][Lp][D]      description-head key codes
//   vpt      fp16 [H][D][lpp]     description-head value codes, transposed
constexpr int kTextSplitMax = 16;   // list shares of a text-row call (nomas_set_text_split bounds it too)
constexpr int kTailCtasMax = 256;   // CTAs of the split last wave of a dense pair-kernel call

struct WsLayout {
    size_t kc, kt, vc, vt, kh, vht, ksl, vsl, kp, vpt, part_o, part_ml, tail_o, tail_ml, total;
};
static WsLayout ws_layout(const nomas_kv_cache *c, int64_t nq, int64_t lt) {
    const auto &d = c->d;
    const int64_t H = d.heads, D = d.head_dim;
    const int64_t frames = d.window_frames > 0 && d.window_frames < d.capacity_frames ? d.window_frames : d.capacity_frames;
    const int64_t lh = frames * d.tokens_per_frame, lhp = round_up(lh, 16);
    const int64_t lpp = round_up(d.head_store_tokens, 16);
    WsLayout w;
    size_t off = 256;   // WsHeader
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) / 256 * 256;
        return o;
    };
    w.kc = take((size_t)H * nq * D * 2);
    w.kt = take((size_t)H * lt * D * 2);
    w.vc = take((size_t)H * D * round_up(nq, 8) * 2);
    w.vt = take((size_t)H * D * round_up(lt, 8) * 2);
    w.kh = take((size_t)H * lh * D * 2);
    w.vht = take((size_t)H * D * lhp * 2);
    w.ksl = take((size_t)H * lhp * 4);
    w.vsl = take((size_t)H * lhp * 4);
    w.kp = take((size_t)H * d.head_store_tokens * D * 2);
    w.vpt = take((size_t)H * D * lpp * 2);
    w.part_o = take((size_t)kTextSplitMax * lt * H * D * 4);    // text-row partials (split calls)
    w.part_ml = take((size_t)kTextSplitMax * H * lt * 8);
    w.tail_o = take((size_t)kTailCtasMax * 2 * kTile * D * 4);    // split last wave (dense pair kernel)
    w.tail_ml = take((size_t)kTailCtasMax * 2 * kTile * 8);
    w.total = off;
    return w;
}

static WsHeader ws_header(const nomas_kv_cache *c, const nomas_mask_layout &lay) {
    WsHeader h{};
    h.magic = kWsMagic;
    h.head_dim = c->d.head_dim;
    h.cache_version = c->version;
    h.head_tokens = lay.head_tokens;
    h.history_tokens = lay.history_tokens;
    h.n_query = lay.n_query;
    h.text_tokens = lay.text_tokens;
    return h;
}


template <int D>
static int launch_attn(const AttnParams &p, dim3 grid, const CUtensorMap *maps, cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   AttnCfg<D>::SMEM);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(attn smem)", (int)e, cudaGetErrorString(e));
        attr_set = true;
    }
    attn_fwd_kernel<D><<<grid, kAttnThreads, AttnCfg<D>::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4],
                                                                      maps[5], maps[6], maps[7], p);
    return check_launch("attn_fwd_kernel launch");
}

static bool strides_ok(int64_t tok_stride, int64_t head_stride) {
    return tok_stride > 0 && head_stride > 0 && tok_stride % 8 == 0 && head_stride % 8 == 0;
}

// Validate nomas_attn_prepare's arguments (nothing is enqueued).
static int check_prepare(const nomas_kv_cache *c, const nomas_segment_text *seg, const void *kcur, const void *vcur,
                         const void *ktxt, const void *vtxt, int64_t tok_stride, int64_t head_stride,
                         const void *workspace, nomas_mask_layout &lay) {
    const int rc = compute_mask_layout(c, seg, NOMAS_MODE_DENSE, 0.25f, &lay);
    if (rc) return rc;
    if (!kcur || !vcur || !workspace || !aligned16(kcur) || !aligned16(vcur) || !aligned16(workspace))
        return NOMAS_EINVAL;
    if (lay.text_tokens > 0 && (!ktxt || !vtxt || !aligned16(ktxt) || !aligned16(vtxt))) return NOMAS_EINVAL;
    if (!strides_ok(tok_stride, head_stride)) return NOMAS_EINVAL;
    return NOMAS_OK;
}

// Validate nomas_attn_run's arguments (nothing is enqueued).
static int check_run(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                     const void *mask_buf, const void *q, int64_t tok_stride, int64_t head_stride,
                     float softmax_scale, const float *out, const float *lse, const void *workspace,
                     nomas_mask_layout &lay) {
    const int rc = compute_mask_layout(c, seg, mode, keep_frac, &lay);
    if (rc) return rc;
    if (!mask_buf || !aligned16(mask_buf)) return NOMAS_EINVAL;
    if (!q || !out || !workspace || !aligned16(q) || !aligned16(out) || !aligned16(workspace)) return NOMAS_EINVAL;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return NOMAS_EINVAL;
    if (!strides_ok(tok_stride, head_stride)) return NOMAS_EINVAL;
    if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return NOMAS_EINVAL;
    return NOMAS_OK;
}

// The pre-pass: fp16 keys, transposed fp16 values, the history's and heads' codes as fp16, and the
// workspace header.
static int enqueue_prepare(const nomas_kv_cache *c, const nomas_mask_layout &lay, const void *kcur,
                           const void *vcur, const void *ktxt, const void *vtxt, int64_t tok_stride,
                           int64_t head_stride, void *workspace, cudaStream_t st) {
    const auto &d = c->d;
    const int D = d.head_dim, H = d.heads;
    const int64_t Nq = lay.n_query, Lt = lay.text_tokens, Lh = lay.history_tokens, Lp = lay.head_tokens;
    const int64_t nqp = round_up(Nq, 8), ltp = round_up(Lt, 8), lhp = round_up(Lh, 16), lpp = round_up(Lp, 16);
    const WsLayout ws = ws_layout(c, Nq, Lt);
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    int *err = static_cast<int *>(c->buf[NOMAS_BUF_ERR]);
    F16Jobs jobs{};
    jobs.H = H;
    jobs.D = D;
    jobs.tok_stride = tok_stride;
    jobs.head_stride = head_stride;
    jobs.err = err;
    jobs.hdr = ws_header(c, lay);
    jobs.hdr_dst = reinterpret_cast<WsHeader *>(wsb);
    jobs.job[jobs.n_jobs++] = F16Job{static_cast<const __nv_bfloat16 *>(kcur), reinterpret_cast<__half *>(wsb + ws.kc), Nq};
    if (Lt > 0)
        jobs.job[jobs.n_jobs++] =
            F16Job{static_cast<const __nv_bfloat16 *>(ktxt), reinterpret_cast<__half *>(wsb + ws.kt), Lt};

    VtJobs vj{};
    vj.H = H;
    vj.D = D;
    vj.tok_stride = tok_stride;
    vj.head_stride = head_stride;
    vj.err = err;
    vj.job[0] = VtJob{static_cast<const __nv_bfloat16 *>(vcur), reinterpret_cast<__half *>(wsb + ws.vc), Nq, nqp};
    vj.job[1] = VtJob{static_cast<const __nv_bfloat16 *>(Lt > 0 ? vtxt : vcur), reinterpret_cast<__half *>(wsb + ws.vt),
                      Lt, ltp};

    if (Lh > 0 || Lp > 0) {
        const HistView hv = hist_view(c);
        HistPrep hp{};
        hp.k8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_K8]);
        hp.v8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_V8]);
        hp.hk8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_HK8]);
        hp.hv8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_HV8]);
        hp.ks = static_cast<const float *>(c->buf[NOMAS_BUF_KS]);
        hp.vs = static_cast<const float *>(c->buf[NOMAS_BUF_VS]);
        hp.hks = static_cast<const float *>(c->buf[NOMAS_BUF_HKS]);
        hp.hvs = static_cast<const float *>(c->buf[NOMAS_BUF_HVS]);
        hp.err = err;
        hp.kh = reinterpret_cast<__half *>(wsb + ws.kh);
        hp.vht = reinterpret_cast<__half *>(wsb + ws.vht);
        hp.kp = reinterpret_cast<__half *>(wsb + ws.kp);
        hp.vpt = reinterpret_cast<__half *>(wsb + ws.vpt);
        hp.ksl = reinterpret_cast<float *>(wsb + ws.ksl);
        hp.vsl = reinterpret_cast<float *>(wsb + ws.vsl);
        hp.hv = hv;
        hp.Lh = Lh;
        hp.lhp = lhp;
        hp.Lp = Lp;
        hp.lpp = lpp;
        hp.head_rows = d.head_store_tokens;
        hp.H = H;
        hp.D = D;
        return launch_prepare(jobs, vj, Lt > 0, nqp > ltp ? nqp : ltp, &hp, st);
    }
    return launch_prepare(jobs, vj, Lt > 0, nqp > ltp ? nqp : ltp, nullptr, st);
}

// The attention kernel over a prepared workspace.
static int enqueue_run(const nomas_kv_cache *c, const nomas_segment_text *seg, const nomas_mask_layout &lay, int mode,
                       const void *mask_buf, const void *q, int64_t tok_stride, int64_t head_stride,
                       float softmax_scale, float *out, float *lse, void *workspace, cudaStream_t st) {
    const auto &d = c->d;
    const int D = d.head_dim, H = d.heads;
    const int64_t Nq = lay.n_query, Lt = lay.text_tokens, Lh = lay.history_tokens, Lp = lay.head_tokens;
    const int64_t nqp = round_up(Nq, 8), ltp = round_up(Lt, 8), lhp = round_up(Lh, 16), lpp = round_up(Lp, 16);
    const WsLayout ws = ws_layout(c, Nq, Lt);
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    // tensor maps (an extent of zero gets a one-row map that no tile reads)
    CUtensorMap maps[8];
    {
        const CUtensorMapDataType F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        const cuuint32_t bk[3] = {64, (cuuint32_t)kTile, 1};        // K: 64 columns x 128 keys
        const cuuint32_t bv[3] = {64, (cuuint32_t)D, 1};            // V^T: 64 keys x D rows
        auto kmap16 = [&](CUtensorMap *m, size_t off, int64_t n) {
            const int64_t nn = n > 0 ? n : 1;
            const cuuint64_t dm[3] = {(cuuint64_t)D, (cuuint64_t)nn, (cuuint64_t)H};
            const cuuint64_t sd[2] = {(cuuint64_t)D * 2, (cuuint64_t)nn * D * 2};
            return make_map(m, F16, wsb + off, dm, sd, bk, CU_TENSOR_MAP_SWIZZLE_128B);
        };
        auto vmap16 = [&](CUtensorMap *m, size_t off, int64_t n, int64_t np) {
            const int64_t nn = n > 0 ? n : 1, pp = np > 0 ? np : 8;
            const cuuint64_t dm[3] = {(cuuint64_t)nn, (cuuint64_t)D, (cuuint64_t)H};
            const cuuint64_t sd[2] = {(cuuint64_t)pp * 2, (cuuint64_t)D * pp * 2};
            return make_map(m, F16, wsb + off, dm, sd, bv, CU_TENSOR_MAP_SWIZZLE_128B);
        };
        if (!kmap16(&maps[0], ws.kc, Nq) || !kmap16(&maps[1], ws.kt, Lt) || !vmap16(&maps[2], ws.vc, Nq, nqp) ||
            !vmap16(&maps[3], ws.vt, Lt, ltp) || !kmap16(&maps[4], ws.kh, Lh) || !kmap16(&maps[5], ws.kp, Lp) ||
            !vmap16(&maps[6], ws.vht, Lh, lhp) || !vmap16(&maps[7], ws.vpt, Lp, lpp))
            return NOMAS_ECUDA;
    }
    AttnParams p{};
    p.ksl = reinterpret_cast<const float *>(wsb + ws.ksl);
    p.vsl = reinterpret_cast<const float *>(wsb + ws.vsl);
    p.hks = static_cast<const float *>(c->buf[NOMAS_BUF_HKS]);
    p.hvs = static_cast<const float *>(c->buf[NOMAS_BUF_HVS]);
    p.hist_stride = lhp;
    p.head_rows = d.head_store_tokens;
    const uint8_t *mb = static_cast<const uint8_t *>(mask_buf);
    p.mask = mb;
    p.lists = reinterpret_cast<const int4 *>(mb + lay.off_list);
    p.counts = reinterpret_cast<const int32_t *>(mb + lay.off_count);
    p.txtwin = reinterpret_cast<const int2 *>(mb + lay.off_txtwin);
    p.expect.magic = kMaskMagic;
    p.expect.mode = mode;
    p.expect.n_qblocks = lay.n_qblocks;
    p.expect.n_lists = lay.n_lists;
    p.expect.history_tokens = lay.history_tokens;
    p.expect.head_tokens = lay.head_tokens;
    p.expect.cache_version = c->version;
    p.expect.n_query = lay.n_query;
    p.expect.text_tokens = lay.text_tokens;
    p.expect.list_cap = lay.list_cap;
    p.expect.keep = lay.keep;
    p.ws_hdr = reinterpret_cast<const WsHeader *>(wsb);
    p.ws_expect = ws_header(c, lay);
    p.sparse = mode == NOMAS_MODE_SPARSE;
    p.text_rows = mode == NOMAS_MODE_TEXT;
    p.head_len = seg->head_len;
    p.n_pairs = (lay.n_qblocks + 1) / 2;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.tok_stride = tok_stride;
    p.head_stride = head_stride;
    p.H = H;
    p.T = d.tokens_per_frame;
    p.divT = make_fastdiv((uint32_t)d.tokens_per_frame);
    p.Nq = mode == NOMAS_MODE_TEXT ? Lt : Nq;   // query rows of this call
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.out = out;
    p.lse = lse;
    p.err = static_cast<int *>(c->buf[NOMAS_BUF_ERR]);
    p.timeout_ns = wait_limit_ns();
    // Text query rows fill few CTAs (ceil(Lt / 128) x H) and their lists differ in length (head rows see
    // all current video, tail rows one window): each list is cut into S shares of equal length, one CTA
    // each, merged by attn_combine_kernel.  S minimises waves x (share length + 24 tiles of fixed CTA
    // cost) + 2 tiles of merge traffic per share, with the list capacity standing in for the length
    // (production segment: 10 x 16 CTAs, 341 entries, S = 4; S = 3 to 5 measured within 1 %, 16 at +19 %).
    int S = 1;
    if (mode == NOMAS_MODE_TEXT && Lt > 0 && lay.list_cap > 0) {
        const int64_t ctas = (int64_t)lay.n_qblocks * H, sms = sm_count(), cap = lay.list_cap;
        int64_t best = 0;
        for (int s = 1; s <= kTextSplitMax && s <= cap; ++s) {
            const int64_t cost = (ctas * s + sms - 1) / sms * ((cap + s - 1) / s + 24) + 2 * s;
            if (s == 1 || cost < best) best = cost, S = s;
        }
        if (text_split_setting() > 0) S = text_split_setting();
    }
    const int share_len = S > 1 ? (int)((lay.list_cap + S - 1) / S) : 0;
    p.share_len = share_len;
    p.part_o = reinterpret_cast<float *>(wsb + ws.part_o);
    p.part_ml = reinterpret_cast<float2 *>(wsb + ws.part_ml);
    const unsigned nz = share_len > 0 ? (unsigned)((lay.list_cap + share_len - 1) / share_len) : 1u;
    // head_dim 128 video rows (dense mode): one CTA per query-block pair (attn_pair_kernel) when that takes
    // fewer SM-waves of work: a pair CTA runs about 1.6 times as long as a block CTA on the same list
    // (measured per list entry: 4570 cycles for the pair's two blocks, 2900 for one block), so few,
    // partly filled waves favour blocks (480 x 832: 3 block waves against 2 pair waves).  The sparse
    // and text-row lists of a pair's two blocks overlap less (each block keeps its own candidates, and
    // text lists are cut into shares): one CTA per block.  nomas_set_attn_kernel overrides the choice.
    const int choice = attn_kernel_setting();
    bool pair = D == 128 && choice == 2;
    if (D == 128 && choice == 0 && mode == NOMAS_MODE_DENSE) {
        const int64_t sms = sm_count();
        const int64_t wb = ((int64_t)lay.n_qblocks * H + sms - 1) / sms;
        const int64_t wp = ((int64_t)p.n_pairs * H + sms - 1) / sms;
        pair = 16 * wp < 10 * wb;
    }
    // The pair kernel walks units (head, pair) head-major.  A dense call whose units leave a partial last
    // wave (production segment: 1664 units on 148 SMs, 36 left over) runs each left-over unit as S
    // shares of its list (S = SMs / left-over units, at most 16), so that the last wave is one wave of
    // short CTAs; attn_combine_tail_kernel merges them (measured: whole lists in the last wave cost
    // about 5 % of the call).
    const int64_t units = (int64_t)p.n_pairs * H;
    p.n_full = (int)units;
    p.n_tail = p.tail_shares = p.tail_len = 0;
    p.tail_o = reinterpret_cast<float *>(wsb + ws.tail_o);
    p.tail_ml = reinterpret_cast<float2 *>(wsb + ws.tail_ml);
    if (pair && mode == NOMAS_MODE_DENSE && share_len == 0) {
        const int64_t sms = sm_count(), rem = units % sms;
        if (units > sms && rem > 0) {
            const int64_t S = std::min<int64_t>(std::min<int64_t>(16, sms / rem),
                                                std::min<int64_t>(kTailCtasMax / rem, lay.list_cap));
            if (S >= 2) {
                p.n_full = (int)(units - rem);
                p.n_tail = (int)rem;
                p.tail_shares = (int)S;
                p.tail_len = (int)((lay.list_cap + S - 1) / S);
            }
        }
    }
    const unsigned pair_ctas = (unsigned)(p.n_full + (int64_t)p.n_tail * p.tail_shares);
    dim3 grid(pair ? pair_ctas : (unsigned)lay.n_qblocks, pair ? 1u : (unsigned)H, nz);
    int rc = pair ? launch_attn_pair(p, grid, maps, st)
             : D == 128 ? launch_attn<128>(p, grid, maps, st) : launch_attn<64>(p, grid, maps, st);
    if (rc) return rc;
    if (p.tail_len > 0) return launch_combine_tail(p, D, st);
    if (share_len == 0) return rc;
    const int64_t warps = Lt * H;
    const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
    if (D == 128)
        attn_combine_kernel<128><<<blocks, 256, 0, st>>>(p.part_o, p.part_ml, p.counts, share_len, Lt, H, out, lse);
    else
        attn_combine_kernel<64><<<blocks, 256, 0, st>>>(p.part_o, p.part_ml, p.counts, share_len, Lt, H, out, lse);
    return check_launch("attn_combine_kernel launch");
}

}  // namespace nomas

using namespace nomas;

extern "C" size_t nomas_attn_workspace_bytes(const nomas_kv_cache *c, const nomas_segment_text *seg) {
    nomas_mask_layout lay;
    if (compute_mask_layout(c, seg, NOMAS_MODE_DENSE, 0.25f, &lay) != NOMAS_OK) return 0;
    return ws_layout(c, lay.n_query, lay.text_tokens).total;
}

extern "C" int nomas_attn_prepare(const nomas_kv_cache *c, const nomas_segment_text *seg, const void *kcur,
                                  const void *vcur, const void *ktxt, const void *vtxt, int64_t tok_stride,
                                  int64_t head_stride, void *workspace, nomas_stream stream) {
    nomas_mask_layout lay;
    const int rc = check_prepare(c, seg, kcur, vcur, ktxt, vtxt, tok_stride, head_stride, workspace, lay);
    if (rc) return rc;
    if (bind_device(c)) return NOMAS_ECUDA;
    return enqueue_prepare(c, lay, kcur, vcur, ktxt, vtxt, tok_stride, head_stride, workspace,
                           reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int nomas_attn_run(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                              const void *mask_buf, const void *q, int64_t tok_stride, int64_t head_stride,
                              float softmax_scale, float *out, float *lse, void *workspace, nomas_stream stream) {
    nomas_mask_layout lay;
    const int rc = check_run(c, seg, mode, keep_frac, mask_buf, q, tok_stride, head_stride, softmax_scale, out, lse,
                             workspace, lay);
    if (rc) return rc;
    if (bind_device(c)) return NOMAS_ECUDA;
    return enqueue_run(c, seg, lay, mode, mask_buf, q, tok_stride, head_stride, softmax_scale, out, lse, workspace,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int nomas_attn_fwd(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                              const void *mask_buf, const void *q, const void *kcur, const void *vcur,
                              const void *ktxt, const void *vtxt, int64_t tok_stride, int64_t head_stride,
                              float softmax_scale, float *out, float *lse, void *workspace, nomas_stream stream) {
    nomas_mask_layout lay_p, lay_r;
    int rc = check_prepare(c, seg, kcur, vcur, ktxt, vtxt, tok_stride, head_stride, workspace, lay_p);
    if (rc) return rc;
    rc = check_run(c, seg, mode, keep_frac, mask_buf, q, tok_stride, head_stride, softmax_scale, out, lse, workspace,
                   lay_r);
    if (rc) return rc;
    if (bind_device(c)) return NOMAS_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = enqueue_prepare(c, lay_p, kcur, vcur, ktxt, vtxt, tok_stride, head_stride, workspace, st))) return rc;
    return enqueue_run(c, seg, lay_r, mode, mask_buf, q, tok_stride, head_stride, softmax_scale, out, lse, workspace,
                       st);
}
