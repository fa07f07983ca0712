// nomas_attn_fwd: action-aware segment-causal attention over an INT8 history (fluxbbs.com "架构" for
// the visibility; "单卡 4090 怎么做到的" for INT8 storage and the sparse mode).
//
// One CTA = one head x two 128-row query tiles (Q0, Q1) that share every K/V tile of their list.
//   warps 0-3   softmax for Q0   (TMEM lanes 0-127 of S0 / O0; one thread per query row)
//   warps 4-7   softmax for Q1
//   warps 8-11  loader: converts Q in place once; TMA for current-segment and text K/V tiles (fp16,
//               prepared by values_f16_kernel); INT8 keys -> fp16 codes and INT8 values x scale ->
//               fp16 written in the 128B-swizzled UMMA layout; per-column key scale and visibility
//               window for the softmax
//   warp 12     tcgen05.mma issuer (one thread) and TMEM owner; warps 13-15 idle
// The register file is split per SM sub-partition (one warp of each warpgroup on each), so the
// kernel launches at 128 registers per thread and moves them with setmaxnreg: softmax 168 each,
// loader 112, MMA warpgroup 64 -- 2*168 + 112 + 64 = 512 = 4 x 128, the launch's own total.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D); P_q (fp16) overwrites
// the first 64 columns of S_q and feeds the PV MMA as its A operand.
//
// Precision: every MMA operand is fp16 with fp32 accumulation.  bf16 inputs convert to fp16
// exactly for magnitudes in [2^-14, 65504] (the supported input range; smaller values keep 2^-24
// absolute resolution), INT8 key codes are exact and the key scale is applied to the fp32 score,
// cached values are fp16(code * scale), and P <= 2^8 keeps 11 significant bits.
//
// Scheduling: per KV tile j the MMA thread issues S_q = Q_q K_j^T when K_j has landed and PV_q of
// the previous tile has been issued, and O_q += P_q V_j when softmax q has published P_q, so the
// tensor core works on one query tile while the other tile's softmax runs.  Softmax uses a lazy
// rescale: the running offset moves only when the row maximum grows by more than 8 (log2 units),
// and then O_q is rescaled in TMEM by its owning thread; completion of S_q(j) implies completion of
// every earlier MMA of this thread (tcgen05.commit tracks all prior operations), so O_q is idle
// whenever softmax q holds a fresh S_q.
#include <cmath>
#include <cstdio>
#include <cuda_fp16.h>

#include "common.cuh"

namespace nomas {

constexpr int kAttnThreads = 512;
constexpr int kRegSoftmax = 168, kRegLoader = 112, kRegMma = 64;
static_assert(2 * kRegSoftmax + kRegLoader + kRegMma == 4 * 128, "register split must equal the launch total");
constexpr int kNCI = 4;                     // column-info ring depth
constexpr float kRescaleThreshold = 8.0f;   // log2 units

template <int D>
struct AttnCfg {
    static constexpr int NS = (D == 128) ? 4 : 8;          // K/V tile slots (K_j, V_j alternate)
    static constexpr int SLOT = kTile * D * 2;             // bytes of one 16-bit tile
    static constexpr int QB = kTile * D * 2;
    static constexpr int HALVES = D / 64;                  // 64-column (128-byte) swizzle panels
    static constexpr int KSTEPS = D / 16;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + 2 * QB;
    static constexpr int OFF_CS = OFF_KV + NS * SLOT;      // float [kNCI][128]
    static constexpr int OFF_CW = OFF_CS + kNCI * 512;     // int2  [kNCI][128]
    static constexpr int OFF_BAR = OFF_CW + kNCI * 1024;
    static constexpr int NBAR = 2 + 2 * NS + 2 * kNCI + 6;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int SMEM = BYTES + 1024;              // slack for 1024-byte alignment
};

struct AttnParams {
    // cached keys / values
    const int8_t *k8, *v8;
    const float *ks, *vs;
    const int8_t *hk8, *hv8;
    const float *hks, *hvs;
    int64_t ring_tokens, first_tok, head_rows;
    // mask buffer
    const uint8_t *mask;
    const int4 *lists;
    const int32_t *counts;
    const int2 *txtwin;
    MaskHeader expect;
    int32_t sparse;
    int32_t n_pairs;
    // shapes
    int32_t H, T;
    int64_t Nq;
    float scale_log2;           // softmax_scale * log2(e)
    float *out;
    float *lse;
    int *err;
    uint64_t timeout_ns;
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t f16x2_of(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// 16 int8 codes -> 16 exact fp16 values (two 16-byte chunks).  Each biased byte u = b + 128 becomes
// the low byte of the fp16 pattern 0x64uu = 1024 + u; one packed add of -1152 leaves b exactly.
__device__ __forceinline__ void i8x16_to_f16(const uint4 &w, uint4 &lo, uint4 &hi) {
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t x = in[i] ^ 0x80808080u;
        o[2 * i] = hadd2_u32(__byte_perm(x, 0x64646464u, 0x4140), 0xE480E480u);
        o[2 * i + 1] = hadd2_u32(__byte_perm(x, 0x64646464u, 0x4342), 0xE480E480u);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// 16 int8 codes times a row scale -> 16 fp16 values.  Each biased byte u becomes the float
// 2^23 + u (pattern 0x4B0000uu); subtracting 2^23 + 128 leaves the code exactly in fp32, which is
// multiplied by the scale and rounded once to fp16.
__device__ __forceinline__ void i8x16_scaled_to_f16(const uint4 &w, float s, uint4 &lo, uint4 &hi) {
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    const float2 bias = make_float2(-8388736.0f, -8388736.0f);
    const float2 sc = make_float2(s, s);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t x = in[i] ^ 0x80808080u;
        float2 a = make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440)),
                               __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7441)));
        float2 b = make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7442)),
                               __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7443)));
        a = __fmul2_rn(__fadd2_rn(a, bias), sc);
        b = __fmul2_rn(__fadd2_rn(b, bias), sc);
        o[2 * i] = f16x2_of(a.x, a.y);
        o[2 * i + 1] = f16x2_of(b.x, b.y);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// 8 bf16 -> 8 fp16 (16 bytes in, 16 bytes out).
__device__ __forceinline__ uint4 bf16x8_to_f16(const uint4 &v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = f16x2_of(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kt,
                    const __grid_constant__ CUtensorMap tm_vt, const AttnParams p) {
    using C = AttnCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t *sQ = sm + C::OFF_Q;
    uint8_t *sKV = sm + C::OFF_KV;
    float *sCS = reinterpret_cast<float *>(sm + C::OFF_CS);
    int2 *sCW = reinterpret_cast<int2 *>(sm + C::OFF_CW);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *bar_q = bars;          // Q tiles landed (TMA, bf16)
    uint64_t *q_ready = bars + 1;    // Q converted to fp16 in place
    uint64_t *kv_full = bars + 2;
    uint64_t *kv_empty = kv_full + C::NS;
    uint64_t *ci_full = kv_empty + C::NS;
    uint64_t *ci_empty = ci_full + kNCI;
    uint64_t *s_full = ci_empty + kNCI;
    uint64_t *p_full = s_full + 2;
    uint64_t *o_final = p_full + 2;
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int pair = blockIdx.x;
    const int h = blockIdx.y;
    const int list_id = p.sparse ? h * p.n_pairs + pair : pair;
    const int4 *list = p.lists + (int64_t)list_id * p.expect.list_cap;

    // header check (every thread reads the same words; all take the same branch)
    const MaskHeader *hd = reinterpret_cast<const MaskHeader *>(p.mask);
    const bool hdr_ok = hd->magic == p.expect.magic && hd->mode == p.expect.mode &&
                        hd->n_qblocks == p.expect.n_qblocks && hd->n_lists == p.expect.n_lists &&
                        hd->history_tokens == p.expect.history_tokens && hd->head_tokens == p.expect.head_tokens &&
                        hd->frames_appended == p.expect.frames_appended && hd->n_query == p.expect.n_query &&
                        hd->text_tokens == p.expect.text_tokens && hd->list_cap == p.expect.list_cap;
    if (!hdr_ok) {
        if (threadIdx.x == 0) set_device_error(p.err, NOMAS_EDEVICE, 1);
        return;
    }
    const int n_tiles = p.counts[list_id];

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(q_ready, 1);
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < kNCI; ++i) {
            mbar_init(&ci_full[i], 1);
            mbar_init(&ci_empty[i], 8);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(&s_full[q], 1);
            mbar_init(&p_full[q], 4);
            mbar_init(&o_final[q], 1);
        }
        misc[1] = 0;
        for (int i = 0; i < C::NS; ++i) misc[8 + i] = 0;
        fence_mbar_init();
    }
    if (warp == 12) {
        tmem_alloc(&misc[0], 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    Watchdog wd{p.err, abort_flag, p.timeout_ns, 0};
    const int64_t qrow0 = (int64_t)pair * 2 * kTile;

    if (warp >= 8 && warp < 12) {
        // ------------------------------------------------------------------ loader warpgroup
        setmaxnreg_dec<kRegLoader>();
        // Every wait is followed by a named barrier over the 128 loader threads and a read of the
        // shared abort flag, so all loader threads leave the loop together.
        wd.where = 3;
        const int t = threadIdx.x - 256;   // 0..127
        uint32_t tma_pending = 0, tma_par = 0;   // per slot: a TMA was issued / its phase parity
        if (t == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_kc);
            prefetch_tmap(&tm_vc);
            mbar_arrive_expect_tx(bar_q, 2 * C::QB);
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int hh = 0; hh < C::HALVES; ++hh)
                    tma_load_3d(sQ + q * C::QB + hh * (kTile * 128), &tm_q, bar_q, hh * 64, h,
                                (int)(qrow0 + q * kTile));
        }
        // Q: bf16 -> fp16 in place (the conversion keeps every element's byte position)
        mbar_wait(bar_q, 0, wd, 4);
        named_bar_sync(1, 128);
        if (!*abort_flag) {
#pragma unroll 4
            for (int i = t; i < 2 * C::QB / 16; i += 128) {
                uint4 *ptr = reinterpret_cast<uint4 *>(sQ) + i;
                *ptr = bf16x8_to_f16(*ptr);
            }
            fence_proxy_async_smem();
        }
        named_bar_sync(1, 128);
        if (t == 0 && !*abort_flag) mbar_arrive(q_ready);

        constexpr int CPR = D / 16;          // 16-byte int8 chunks per row
        constexpr int RSTEP = 128 / CPR;     // rows covered by the 128 threads in one pass
        constexpr int NR = 128 / RSTEP;      // rows per thread
        const int my_chunk = t % CPR;
        const int my_row0 = t / CPR;
        const int hh_mine = my_chunk / 4;
        const int c0_mine = (my_chunk % 4) * 2;
        for (int j = 0; j < n_tiles && !*abort_flag; ++j) {
            const int4 e = list[j];
            const int kind = e.x & 3;
            const int64_t start = e.y;
            const int count = e.z;
            const bool cached = kind == kKindHist || kind == kKindPriorHead;
            const bool hist = kind == kKindHist;
            const int8_t *src_k = hist ? p.k8 : p.hk8;
            const int8_t *src_v = hist ? p.v8 : p.hv8;
            const float *src_ks = hist ? p.ks : p.hks;
            const float *src_vs = hist ? p.vs : p.hvs;
            const int64_t head_base = (int64_t)h * (hist ? p.ring_tokens : p.head_rows);
            auto cache_row = [&](int r) -> int64_t {  // head-major row index of tile row r
                const int64_t a = start + r;
                return head_base + (hist ? (p.first_tok + a) % p.ring_tokens : a);
            };
            // raw INT8 loads issued first so that their latency overlaps the slot waits
            uint4 rk[NR], rv[NR];
            float svv[NR];
            if (cached) {
#pragma unroll
                for (int i = 0; i < NR; ++i) {
                    const int r = my_row0 + i * RSTEP;
                    rk[i] = rv[i] = make_uint4(0, 0, 0, 0);
                    svv[i] = 0.0f;
                    if (r < count) {
                        const int64_t gr = cache_row(r);
                        rk[i] = __ldg(reinterpret_cast<const uint4 *>(src_k + gr * D) + my_chunk);
                        rv[i] = __ldg(reinterpret_cast<const uint4 *>(src_v + gr * D) + my_chunk);
                        svv[i] = __ldg(src_vs + gr);
                    }
                }
            }
            float cs = 0.0f;
            int2 w = make_int2(kAlwaysHi, 0);
            if (t < count) {
                w = kind == kKindText ? p.txtwin[start + t] : make_int2(0, kAlwaysHi);
                cs = cached ? __ldg(src_ks + cache_row(t)) * p.scale_log2 : p.scale_log2;
            }
            const int ci = j % kNCI;
            const int sk = (2 * j) % C::NS;
            const int sv = (2 * j + 1) % C::NS;
            if (mbar_wait(&ci_empty[ci], ((j / kNCI) & 1) ^ 1, wd, 1))
                mbar_wait(&kv_empty[sk], (((2 * j) / C::NS) & 1) ^ 1, wd, 2);
            named_bar_sync(1, 128);
            if (*abort_flag) break;
            sCS[ci * 128 + t] = cs;
            sCW[ci * 128 + t] = w;
            uint8_t *dK = sKV + sk * C::SLOT;
            if (!cached) {
                if (t == 0) {
                    const CUtensorMap *m = kind == kKindCur ? &tm_kc : &tm_kt;
                    mbar_arrive_expect_tx(&kv_full[sk], C::SLOT);
#pragma unroll
                    for (int hh = 0; hh < C::HALVES; ++hh)
                        tma_load_3d(dK + hh * (kTile * 128), m, &kv_full[sk], hh * 64, (int)start, h);
                    tma_pending |= 1u << sk;
                    tma_par = (tma_par & ~(1u << sk)) | ((uint32_t)(((2 * j) / C::NS) & 1) << sk);
                }
            } else {
#pragma unroll
                for (int i = 0; i < NR; ++i) {
                    const int r = my_row0 + i * RSTEP;
                    uint4 lo, hi;
                    i8x16_to_f16(rk[i], lo, hi);
                    uint8_t *base = dK + hh_mine * (kTile * 128);
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, c0_mine)) = lo;
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, c0_mine + 1)) = hi;
                }
                fence_proxy_async_smem();
                tma_pending &= ~(1u << sk);
            }
            named_bar_sync(1, 128);
            if (t == 0) {
                mbar_arrive(&ci_full[ci]);
                if (cached) mbar_arrive(&kv_full[sk]);
            }
            mbar_wait(&kv_empty[sv], (((2 * j + 1) / C::NS) & 1) ^ 1, wd, 3);
            named_bar_sync(1, 128);
            if (*abort_flag) break;
            uint8_t *dV = sKV + sv * C::SLOT;
            if (!cached) {
                if (t == 0) {
                    const CUtensorMap *m = kind == kKindCur ? &tm_vc : &tm_vt;
                    mbar_arrive_expect_tx(&kv_full[sv], C::SLOT);
#pragma unroll
                    for (int hh = 0; hh < C::HALVES; ++hh)
                        tma_load_3d(dV + hh * (kTile * 128), m, &kv_full[sv], hh * 64, (int)start, h);
                    tma_pending |= 1u << sv;
                    tma_par = (tma_par & ~(1u << sv)) | ((uint32_t)(((2 * j + 1) / C::NS) & 1) << sv);
                }
            } else {
#pragma unroll
                for (int i = 0; i < NR; ++i) {
                    const int r = my_row0 + i * RSTEP;
                    uint4 lo, hi;
                    i8x16_scaled_to_f16(rv[i], svv[i], lo, hi);
                    uint8_t *base = dV + hh_mine * (kTile * 128);
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, c0_mine)) = lo;
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, c0_mine + 1)) = hi;
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                tma_pending &= ~(1u << sv);
                if (t == 0) mbar_arrive(&kv_full[sv]);
            }
        }
        // on abort, let this CTA's bulk copies land before the shared memory is released
        if (*abort_flag && t == 0) {
            mbar_drain(bar_q, 0, 100000000ull);
#pragma unroll
            for (int i = 0; i < C::NS; ++i)
                if ((tma_pending >> i) & 1u) mbar_drain(&kv_full[i], (tma_par >> i) & 1u, 100000000ull);
        }
    } else if (warp >= 12) {
        // ------------------------------------------------------------------ MMA issuer (warp 12)
        setmaxnreg_dec<kRegMma>();
        wd.where = 4;
        if (warp == 12 && lane == 0) {
            constexpr uint32_t idesc_qk = idesc_f16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_f16_f32(128, D, false, true);
            const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
            const uint32_t tO[2] = {tmem + 256u, tmem + 384u};
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t kv_addr = smem_u32(sKV);
            bool ok = mbar_wait(q_ready, 0, wd, 1);
            int next_s[2];              // next list index whose S_q is to be issued
            int pend[2] = {-1, -1};     // list index whose PV_q waits for P_q
            int last_s[2] = {-1, -1}, last_pv[2] = {-1, -1};
            uint32_t pcount[2] = {0, 0};
            bool first_pv[2] = {true, true};
            auto uses = [&](int j, int q) -> bool { return (list[j].x & (q ? kUse1 : kUse0)) != 0; };
            auto advance = [&](int j, int q) -> int {
                while (j < n_tiles && !uses(j, q)) ++j;
                return j;
            };
            next_s[0] = advance(0, 0);
            next_s[1] = advance(0, 1);
            // released[s]: how many uses of K/V slot s this thread has released.  A slot is tested
            // for use u only when uses 0..u-1 are released, so its full barrier can only be at phase
            // u or u+1 and the parity test cannot mistake an older completion for use u.
            uint32_t *released = misc + 8;
            uint64_t t0 = globaltimer_ns();
            uint32_t spins = 0;
            while (ok && (next_s[0] < n_tiles || next_s[1] < n_tiles || pend[0] >= 0 || pend[1] >= 0)) {
                bool progress = false;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    if (pend[q] >= 0) {
                        const int j = pend[q];
                        const int sv = (2 * j + 1) % C::NS;
                        const uint32_t use_v = (uint32_t)((2 * j + 1) / C::NS);
                        if (released[sv] == use_v && mbar_test(&p_full[q], pcount[q] & 1) &&
                            mbar_test(&kv_full[sv], use_v & 1)) {
                            tc_fence_after();
                            const uint32_t vb = kv_addr + sv * C::SLOT;
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t bdesc = sdesc_sw128(vb + kk * 16 * 128, kTile * 128, 1024);
                                umma_ts(tO[q], tS[q] + kk * 8, bdesc, idesc_pv, (kk > 0 || !first_pv[q]) ? 1u : 0u);
                            }
                            first_pv[q] = false;
                            pcount[q]++;
                            last_pv[q] = j;
                            const int o = 1 - q;
                            if (!uses(j, o) || last_pv[o] >= j) {
                                umma_commit(&kv_empty[sv]);
                                released[sv] = use_v + 1;
                            }
                            pend[q] = -1;
                            progress = true;
                        }
                    }
                    if (pend[q] < 0 && next_s[q] < n_tiles) {
                        const int j = next_s[q];
                        const int sk = (2 * j) % C::NS;
                        const uint32_t use_k = (uint32_t)((2 * j) / C::NS);
                        if (released[sk] == use_k && mbar_test(&kv_full[sk], use_k & 1)) {
                            tc_fence_after();
                            const uint32_t kb = kv_addr + sk * C::SLOT;
                            const uint32_t qb = q_addr + q * C::QB;
#pragma unroll
                            for (int kk = 0; kk < C::KSTEPS; ++kk) {
                                const uint32_t off = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
                                umma_ss(tS[q], sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                                        idesc_qk, kk > 0 ? 1u : 0u);
                            }
                            umma_commit(&s_full[q]);
                            last_s[q] = j;
                            const int o = 1 - q;
                            if (!uses(j, o) || last_s[o] >= j) {
                                umma_commit(&kv_empty[sk]);
                                released[sk] = use_k + 1;
                            }
                            pend[q] = j;
                            next_s[q] = advance(j + 1, q);
                            progress = true;
                        }
                    }
                }
                if (progress) {
                    spins = 0;
                    t0 = globaltimer_ns();
                } else if (++spins > 64) {
                    spins = 0;
                    if (*abort_flag) ok = false;
                    else if (globaltimer_ns() - t0 > p.timeout_ns) {
                        set_device_error(p.err, NOMAS_ETIMEOUT, 405);
                        *abort_flag = 1;
                        ok = false;
                    }
                }
            }
            umma_commit(&o_final[0]);
            umma_commit(&o_final[1]);
            // the MMAs must be complete before the CTA releases TMEM, also on the abort path
            if (!ok) mbar_drain(&o_final[1], 0, 100000000ull);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax warpgroups
        // Waits are made warp-uniform (__all_sync) because tcgen05.ld/st are warp-collective.
        setmaxnreg_inc<kRegSoftmax>();
        const int q = warp >> 2;
        wd.where = 1 + q;
        const int r = (warp & 3) * 32 + lane;
        const int64_t row = qrow0 + q * kTile + r;
        const int frame = (int)((row < p.Nq ? row : 0) / p.T);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + (uint32_t)(q * 128);
        const uint32_t tO = tmem + lane_base + 256u + (uint32_t)(q * 128);
        float m_used = -INFINITY;
        float l = 0.0f;
        uint32_t k = 0;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int4 e = list[j];
            const int ci = j % kNCI;
            ok = __all_sync(0xffffffffu, mbar_wait(&ci_full[ci], (j / kNCI) & 1, wd, 1));
            if (!ok) break;
            const bool used = (e.x & (q ? kUse1 : kUse0)) != 0;
            if (!used) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&ci_empty[ci]);
                continue;
            }
            const bool masked = (e.x & (q ? kMask1 : kMask0)) != 0;
            const bool cached = (e.x & 3) == kKindHist || (e.x & 3) == kKindPriorHead;
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[q], k & 1, wd, 2));
            if (!ok) break;
            tc_fence_after();
            float s[128];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) tmem_ld32f_sync(tS + c4 * 32, &s[c4 * 32]);
            // cached keys: apply the per-key scale (which carries softmax scale * log2 e) to the score
            if (cached) {
                const float4 *cs4 = reinterpret_cast<const float4 *>(sCS + ci * 128);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if ((i & 7) == 0) asm volatile("" ::: "memory");   // bound how far loads are hoisted
                    const float4 v = cs4[i];
                    const float2 a = __fmul2_rn(make_float2(s[4 * i], s[4 * i + 1]), make_float2(v.x, v.y));
                    const float2 b = __fmul2_rn(make_float2(s[4 * i + 2], s[4 * i + 3]), make_float2(v.z, v.w));
                    s[4 * i] = a.x;
                    s[4 * i + 1] = a.y;
                    s[4 * i + 2] = b.x;
                    s[4 * i + 3] = b.y;
                }
            }
            if (masked) {
                const int4 *cw = reinterpret_cast<const int4 *>(sCW + ci * 128);
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    if ((i & 7) == 0) asm volatile("" ::: "memory");
                    const int4 w = cw[i];   // windows of columns 2i and 2i+1
                    s[2 * i] = (w.x <= frame && frame < w.y) ? s[2 * i] : -INFINITY;
                    s[2 * i + 1] = (w.z <= frame && frame < w.w) ? s[2 * i + 1] : -INFINITY;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ci_empty[ci]);
            float mt = max3(s[0], s[1], s[2]);
#pragma unroll
            for (int c = 3; c < 127; c += 2) mt = max3(mt, s[c], s[c + 1]);
            mt = fmaxf(mt, s[127]);
            // log2 domain: cached scores are already scaled, bf16-source scores get the uniform scale
            const float cmul = cached ? 1.0f : p.scale_log2;
            mt *= cmul;
            const float m_new = fmaxf(m_used, mt);
            const bool grow = m_new > m_used + kRescaleThreshold;   // false while both are -inf
            const bool need_o = grow && m_used != -INFINITY;
            const float f = need_o ? ex2(m_used - m_new) : 1.0f;
            if (grow) m_used = m_new;
            const float off = (m_used == -INFINITY) ? 0.0f : m_used;
            const float2 cm2 = make_float2(cmul, cmul);
            const float2 no2 = make_float2(-off, -off);
            float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int qt = 0; qt < 4; ++qt) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 a = __ffma2_rn(make_float2(s[qt * 32 + c], s[qt * 32 + c + 1]), cm2, no2);
                    const float p0 = ex2(a.x);
                    const float p1 = ex2(a.y);
                    acc = __fadd2_rn(acc, make_float2(p0, p1));
                    pk[c / 2] = f16x2_of(p0, p1);
                }
                tmem_st16(tS + qt * 16, pk);
            }
            l = l * f + (acc.x + acc.y);
            // rescale O_q in TMEM (rare: only when some row's maximum grew past the threshold);
            // done after P so that the scores are no longer live
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
            if (lane == 0) mbar_arrive(&p_full[q]);
            ++k;
        }
        // epilogue: O / l
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_final[q], 0, wd, 3));
        if (ok) {
            tc_fence_after();
            const float inv = l > 0.0f ? 1.0f / l : 0.0f;
            float *dst = p.out + (row * p.H + h) * (int64_t)D;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t rr[32];
                tmem_ld32_sync(tO + c0, rr);
                if (row < p.Nq) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 v = make_float4(__uint_as_float(rr[i]) * inv, __uint_as_float(rr[i + 1]) * inv,
                                                     __uint_as_float(rr[i + 2]) * inv, __uint_as_float(rr[i + 3]) * inv);
                        *reinterpret_cast<float4 *>(dst + c0 + i) = v;
                    }
                }
            }
            if (p.lse && row < p.Nq)
                p.lse[(int64_t)h * p.Nq + row] = (m_used + log2f(l)) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// bf16 [n][H][D] (token / head strides in elements) -> fp16 [H][n][D], for up to four tensors.
struct F16Job {
    const __nv_bfloat16 *src;
    __half *dst;
    int64_t n;
};
struct F16Jobs {
    F16Job job[4];
    int32_t n_jobs;
    int32_t H, D;
    int64_t tok_stride, head_stride;
};

__global__ void __launch_bounds__(256) values_f16_kernel(F16Jobs jobs) {
    const int cpr = jobs.D / 8;   // 16-byte chunks per row
    for (int jb = 0; jb < jobs.n_jobs; ++jb) {
        const F16Job J = jobs.job[jb];
        const int64_t total = J.n * jobs.H * cpr;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
             i += (int64_t)gridDim.x * blockDim.x) {
            const int c = (int)(i % cpr);
            const int64_t rowi = i / cpr;              // = h * n + t  (destination order)
            const int64_t t = rowi % J.n;
            const int h = (int)(rowi / J.n);
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(J.src + t * jobs.tok_stride +
                                                                  (int64_t)h * jobs.head_stride) + c);
            reinterpret_cast<uint4 *>(J.dst + rowi * jobs.D)[c] = bf16x8_to_f16(v);
        }
    }
}

}  // namespace nomas

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
namespace nomas {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr = cudaDriverEntryPointSymbolNotFound;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr);
        if (e == cudaSuccess && qr == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(ptr);
        else cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", e != cudaSuccess ? (int)e : (int)qr,
                       e != cudaSuccess ? cudaGetErrorString(e) : "symbol query failed");
    }
    return fn;
}

// 3-D tiled map with 128B swizzle.  dims / strides are innermost first (strides in bytes for
// dims 1 and 2); the box's inner extent is 64 elements (128 bytes).
static bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, const cuuint64_t dims[3],
                     const cuuint64_t strides[2], const cuuint32_t box[3]) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint32_t es[3] = {1, 1, 1};
    const CUresult r = enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char msg[160];
        std::snprintf(msg, sizeof(msg), "dims %llu x %llu x %llu, strides %llu %llu", (unsigned long long)dims[0],
                      (unsigned long long)dims[1], (unsigned long long)dims[2], (unsigned long long)strides[0],
                      (unsigned long long)strides[1]);
        cuda_fail("cuTensorMapEncodeTiled", (int)r, msg);
        return false;
    }
    return true;
}

// Workspace: fp16 [H][n][D] copies of the current segment's K, V and the text's K, V.
struct WsLayout {
    size_t off[4];
    size_t total;
};
static WsLayout ws_layout(const nomas_kv_cache *c, int64_t nq, int64_t lt) {
    WsLayout w;
    const size_t row = (size_t)c->d.heads * c->d.head_dim * 2;
    size_t off = 0;
    const int64_t n[4] = {nq, nq, lt, lt};
    for (int i = 0; i < 4; ++i) {
        w.off[i] = off;
        off += ((size_t)n[i] * row + 255) / 256 * 256;
    }
    w.total = off;
    return w;
}

static uint64_t g_timeout_ns = 2000000000ull;   // 2 s per wait

template <int D>
static int launch_attn(const AttnParams &p, dim3 grid, const CUtensorMap *maps, cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   AttnCfg<D>::SMEM);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(attn smem)", (int)e, cudaGetErrorString(e));
        attr_set = true;
    }
    attn_fwd_kernel<D><<<grid, kAttnThreads, AttnCfg<D>::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p);
    return check_launch("attn_fwd_kernel launch");
}

}  // namespace nomas

using namespace nomas;

extern "C" size_t nomas_attn_workspace_bytes(const nomas_kv_cache *c, const nomas_segment_text *seg) {
    nomas_mask_layout lay;
    if (compute_mask_layout(c, seg, NOMAS_MODE_DENSE, 0.25f, &lay) != NOMAS_OK) return 0;
    return ws_layout(c, lay.n_query, lay.text_tokens).total;
}

extern "C" int nomas_attn_fwd(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                              const void *mask_buf, const void *q, const void *kcur, const void *vcur,
                              const void *ktxt, const void *vtxt, int64_t tok_stride, int64_t head_stride,
                              float softmax_scale, float *out, float *lse, void *workspace, nomas_stream stream) {
    nomas_mask_layout lay;
    int rc = compute_mask_layout(c, seg, mode, keep_frac, &lay);
    if (rc) return rc;
    if (!mask_buf || !aligned16(mask_buf)) return NOMAS_EINVAL;
    if (!q || !kcur || !vcur || !out || !workspace) return NOMAS_EINVAL;
    if (!aligned16(q) || !aligned16(kcur) || !aligned16(vcur) || !aligned16(out) || !aligned16(workspace))
        return NOMAS_EINVAL;
    if (lay.text_tokens > 0 && (!ktxt || !vtxt || !aligned16(ktxt) || !aligned16(vtxt))) return NOMAS_EINVAL;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return NOMAS_EINVAL;
    if (tok_stride <= 0 || head_stride <= 0 || tok_stride % 8 || head_stride % 8) return NOMAS_EINVAL;
    if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return NOMAS_EINVAL;
    const auto &d = c->d;
    const int D = d.head_dim;
    const int H = d.heads;
    if (bind_device(c)) return NOMAS_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    // fp16 copies of the current segment's and the text's K / V (HBM-bound pre-pass)
    const WsLayout ws = ws_layout(c, lay.n_query, lay.text_tokens);
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    F16Jobs jobs{};
    jobs.H = H;
    jobs.D = D;
    jobs.tok_stride = tok_stride;
    jobs.head_stride = head_stride;
    const void *srcs[4] = {kcur, vcur, ktxt, vtxt};
    const int64_t ns[4] = {lay.n_query, lay.n_query, lay.text_tokens, lay.text_tokens};
    for (int i = 0; i < 4; ++i) {
        if (ns[i] == 0) continue;
        F16Job &J = jobs.job[jobs.n_jobs++];
        J.src = static_cast<const __nv_bfloat16 *>(srcs[i]);
        J.dst = reinterpret_cast<__half *>(wsb + ws.off[i]);
        J.n = ns[i];
    }
    {
        const int64_t chunks = (2 * lay.n_query + 2 * lay.text_tokens) * H * (D / 8);
        int64_t blocks = (chunks + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        values_f16_kernel<<<(unsigned)blocks, 256, 0, st>>>(jobs);
        rc = check_launch("values_f16_kernel launch");
        if (rc) return rc;
    }

    CUtensorMap maps[5];
    {
        const cuuint64_t dq[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)lay.n_query};
        const cuuint64_t sq[2] = {(cuuint64_t)head_stride * 2, (cuuint64_t)tok_stride * 2};
        const cuuint32_t bq[3] = {64, 1, (cuuint32_t)kTile};
        if (!make_map(&maps[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, dq, sq, bq)) return NOMAS_ECUDA;
        const cuuint32_t bk[3] = {64, (cuuint32_t)kTile, 1};
        for (int i = 0; i < 4; ++i) {
            const int64_t n = ns[i] > 0 ? ns[i] : 1;
            const size_t off = ns[i] > 0 ? ws.off[i] : ws.off[0];
            const cuuint64_t dk[3] = {(cuuint64_t)D, (cuuint64_t)n, (cuuint64_t)H};
            const cuuint64_t sk[2] = {(cuuint64_t)D * 2, (cuuint64_t)n * D * 2};
            if (!make_map(&maps[1 + i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, wsb + off, dk, sk, bk)) return NOMAS_ECUDA;
        }
    }
    const HistView hv = hist_view(c);
    AttnParams p{};
    p.k8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_K8]);
    p.v8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_V8]);
    p.ks = static_cast<const float *>(c->buf[NOMAS_BUF_KS]);
    p.vs = static_cast<const float *>(c->buf[NOMAS_BUF_VS]);
    p.hk8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_HK8]);
    p.hv8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_HV8]);
    p.hks = static_cast<const float *>(c->buf[NOMAS_BUF_HKS]);
    p.hvs = static_cast<const float *>(c->buf[NOMAS_BUF_HVS]);
    p.ring_tokens = hv.ring_tokens;
    p.first_tok = hv.first_tok;
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
    p.expect.frames_appended = c->frames_appended;
    p.expect.n_query = lay.n_query;
    p.expect.text_tokens = lay.text_tokens;
    p.expect.list_cap = lay.list_cap;
    p.expect.keep = lay.keep;
    p.sparse = mode == NOMAS_MODE_SPARSE;
    p.n_pairs = (lay.n_qblocks + 1) / 2;
    p.H = H;
    p.T = d.tokens_per_frame;
    p.Nq = lay.n_query;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.out = out;
    p.lse = lse;
    p.err = static_cast<int *>(c->buf[NOMAS_BUF_ERR]);
    p.timeout_ns = g_timeout_ns;
    dim3 grid((unsigned)p.n_pairs, (unsigned)H);
    return D == 128 ? launch_attn<128>(p, grid, maps, st) : launch_attn<64>(p, grid, maps, st);
}
