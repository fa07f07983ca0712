// nomas_kv_append / nomas_kv_dequant: INT8 quantise-append of a finished segment's K/V into the
// sliding-window ring (fluxbbs.com "单卡 4090 怎么做到的", first and second techniques: INT8
// storage with float scales; 18 retained history latent frames) and the description-head store.
//
// HBM-bound: per (token, head) 2*D bf16 read, 2*D int8 + 2 fp32 written.  A persistent kernel: in
// every CTA a producer warp keeps TMA copies of (one head x TC tokens) chunks of K and V in flight
// through a three-stage shared-memory ring while eight consumer warps quantise the chunks already
// landed, so loads overlap the arithmetic.  One group of D/16 lanes handles one (token, head): each
// lane holds 16 channels of K and 16 of V, the absmax is reduced with xor-shuffles inside the group,
// and each lane stores 16 codes.  The ring rows of the video frames and the description-head rows
// are two jobs of the same launch.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "quant.cuh"

namespace nomas {

// max(a, b, c); a NaN operand is ignored unless all three are NaN (PTX max.f32 semantics).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int LPV>
__device__ __forceinline__ float group_max(float a) {
#pragma unroll
    for (int off = LPV / 2; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    return a;
}

__device__ __forceinline__ void unpack16(const uint4 &w0, const uint4 &w1, float (&x)[16]) {
    const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(u[i] << 16);
        x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

// Codes rint(x / s) in fp32 with IEEE division and round-half-even for the 16 channels this lane
// holds; s = RN(absmax / 127) over the group's D channels, so |x / s| <= 127 (1 + 2^-23) and every
// code lies in [-127, 127].
// With r = 1/s to relative 2^-24 + 2^-40, the exact product x r is within 127 (2^-24 + 2^-40) (1 + 2^-23)
// < 2^-17 of x / s, which is within 2^-18 of RN(x / s).  t = RN(x r + 1.5 * 2^23) (one FMA) holds the
// integer q nearest x r, and d = RN(x r - q) (one FMA; |x r - q| <= 1/2, rounding error <= 2^-26).  When
// |d| < 1/2 - 2^-15, RN(x / s) is within 1/2 - 2^-15 + 2^-26 + 2^-17 + 2^-18 < 1/2 of q, so
// rint(RN(x / s)) = q.  Otherwise the exact quotient decides: rarely, and always for s below 2^-125,
// where r is a NaN.  The warp takes that branch only when one of its lanes needs it.  The fp32 add of
// 1.5 * 2^23 leaves q, as a two's-complement byte, in the low byte of t's bit pattern.  The absmax
// and the largest |d| of the lane are taken with three-input maxima (which return a NaN only when every
// operand is one, so a NaN start value drops out and an all-NaN d -- the tiny-s case -- stays NaN).
template <int LPV>
__device__ __forceinline__ uint4 quant16(const float (&x)[16], float &s_out) {
    constexpr float kMagic = 12582912.0f;                 // 1.5 * 2^23
    constexpr float kFar = 0.5f - 0x1p-15f;               // |y - rint(y)| below this: not near a tie
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i += 2) a = max3f(a, fabsf(x[i]), fabsf(x[i + 1]));
    a = group_max<LPV>(a);
    const float s = div127(a);
    s_out = s;
    const bool nz = s > 0.0f;
    const float r = s >= 0x1p-125f ? recip_nr(s) : (nz ? __int_as_float(0x7fffffff) : 0.0f);
    const float2 r2 = make_float2(r, r), m2 = make_float2(kMagic, kMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    uint32_t tb[16];
    float dmax = __int_as_float(0x7fffffff);             // NaN: max.f32 keeps the other operands
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 xx = make_float2(x[2 * i], x[2 * i + 1]);
        const float2 t = __ffma2_rn(xx, r2, m2);
        const float2 nq = __ffma2_rn(t, neg1, m2);
        const float2 d = __ffma2_rn(xx, r2, nq);
        dmax = max3f(dmax, fabsf(d.x), fabsf(d.y));
        tb[2 * i] = __float_as_uint(t.x);
        tb[2 * i + 1] = __float_as_uint(t.y);
    }
    const bool slow = !(dmax < kFar);                     // NaN (tiny s: every d is NaN) counts as near
    if (__any_sync(0xffffffffu, slow && nz)) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float t = __fmaf_rn(x[i], r, kMagic);
            const float d = __fmaf_rn(x[i], r, -__fsub_rn(t, kMagic));
            if (nz && !(fabsf(d) < kFar)) tb[i] = __float_as_uint(__fadd_rn(rintf(__fdiv_rn(x[i], s)), kMagic));
        }
    }
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)   // low bytes of t[4i .. 4i+3]
        w[i] = __byte_perm(__byte_perm(tb[4 * i], tb[4 * i + 1], 0x0040), __byte_perm(tb[4 * i + 2], tb[4 * i + 3], 0x0040),
                           0x5410);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int D>
constexpr int kTokBlock = 32 / (D / 16);    // tokens per warp: one token per group of D/16 lanes

constexpr int kAppendConsumers = 8;         // consumer warps; warp 8 is the producer
constexpr int kAppendThreads = 32 * (kAppendConsumers + 1);
constexpr int kAppendStages = 3;          // with four CTAs per SM: 192 KB of chunks in flight per SM

template <int D>
struct AppendCfg {
    static constexpr int TC = kAppendConsumers * kTokBlock<D>;   // tokens per chunk (32 or 64)
    static constexpr int TILE = TC * D * 2;                      // bytes of one K (or V) tile: 8 KB
    static constexpr int STAGE = 2 * TILE;
    static constexpr int OFF_BAR = kAppendStages * STAGE;
    static constexpr int SMEM = OFF_BAR + 2 * kAppendStages * 8 + 1024;   // + slack for 1024-byte alignment
};

// One destination of the append: the newest frames into the ring (video) or the head store.
struct AppendJob {
    int64_t n_tok;            // tokens
    int64_t n_chunks;         // ceil(n_tok / TC) * heads
    int32_t head_mode;        // 0: ring rows slot(frame) * T + r; 1: rows dst_row0 + t
    int32_t first_slot;       // ring slot of the job's first frame (video)
    int32_t tok_outer;        // source maps are (D, heads, tokens) when set, else (D, tokens, heads)
    int32_t use_slots;        // video: frame f goes to slots[f] instead of first_slot + f (mod C)
    int32_t slots[NOMAS_MAX_SELECT_FRAMES];
    int64_t dst_row0;
    int64_t rows_per_head;    // destination rows per head
    int8_t *k8, *v8;
    float *ks, *vs;
};

struct AppendParams {
    AppendJob job[2];
    int32_t heads, tokens_per_frame, capacity_frames;
    FastDiv div_heads, div_frame;     // by heads, by tokens_per_frame
    int *err;
    uint64_t timeout_ns;
};

// Chunk c of the launch (every count below 2^31): job, head and token block (token blocks outer,
// heads inner).
__device__ __forceinline__ void chunk_of(const AppendParams &a, uint32_t c, int &job, int &h, int &tb) {
    job = c < (uint32_t)a.job[0].n_chunks ? 0 : 1;
    if (job) c -= (uint32_t)a.job[0].n_chunks;
    tb = (int)fdiv(c, a.div_heads);
    h = (int)c - tb * a.heads;
}

template <int D>
__global__ void __launch_bounds__(kAppendThreads, 4)
    quant_append_kernel(const __grid_constant__ CUtensorMap tk0, const __grid_constant__ CUtensorMap tv0,
                        const __grid_constant__ CUtensorMap tk1, const __grid_constant__ CUtensorMap tv1,
                        const AppendParams a) {
    using C = AppendCfg<D>;
    constexpr int LPV = D / 16;             // lanes per (token, head) vector
    constexpr int TB = kTokBlock<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR), *empty = full + kAppendStages;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kAppendStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kAppendConsumers);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    Watchdog wd{a.err, &abort_flag, a.timeout_ns, 7};
    const int64_t total = a.job[0].n_chunks + a.job[1].n_chunks;

    if (warp == kAppendConsumers) {
        // ---------------------------------------------------------------- producer (one thread)
        if (lane == 0) {
            uint32_t pend = 0, wpar = 0;    // per stage: a copy was issued, parity of the phase it completes
            int i = 0;
            for (int64_t c = blockIdx.x; c < total; c += gridDim.x, ++i) {
                const int st = i % kAppendStages;
                if (!mbar_wait(&empty[st], ((i / kAppendStages) & 1) ^ 1, wd, 1)) break;
                int job, h, tb;
                chunk_of(a, (uint32_t)c, job, h, tb);
                uint8_t *dk = sm + st * C::STAGE;
                const int y = a.job[job].tok_outer ? h : tb * C::TC;
                const int z = a.job[job].tok_outer ? tb * C::TC : h;
                mbar_arrive_expect_tx(&full[st], C::STAGE);
                tma_load_3d(dk, job ? &tk1 : &tk0, &full[st], 0, y, z);
                tma_load_3d(dk + C::TILE, job ? &tv1 : &tv0, &full[st], 0, y, z);
                pend |= 1u << st;
                wpar = (wpar & ~(1u << st)) | ((uint32_t)((i / kAppendStages) & 1) << st);
            }
            // the copies must land before the CTA's shared memory is released (a no-op unless aborting)
            for (int st = 0; st < kAppendStages; ++st)
                if ((pend >> st) & 1u) mbar_drain(&full[st], (wpar >> st) & 1u, 100000000ull);
        }
        return;
    }
    // -------------------------------------------------------------------- consumers
    const int sub = lane % LPV;
    const int grp = lane / LPV;
    const int T = a.tokens_per_frame, Cf = a.capacity_frames;
    int i = 0;
    for (int64_t c = blockIdx.x; c < total; c += gridDim.x, ++i) {
        const int st = i % kAppendStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (i / kAppendStages) & 1, wd, 2))) break;
        int job, h, tb;
        chunk_of(a, (uint32_t)c, job, h, tb);
        const AppendJob &J = a.job[job];
        const int row_in_chunk = warp * TB + grp;
        const int t = tb * C::TC + row_in_chunk;       // token within the job
        const uint4 *sk = reinterpret_cast<const uint4 *>(sm + st * C::STAGE + row_in_chunk * D * 2 + sub * 32);
        const uint4 *sv = reinterpret_cast<const uint4 *>(sm + st * C::STAGE + C::TILE + row_in_chunk * D * 2 + sub * 32);
        float x[16];
        float skale, svale;
        unpack16(sk[0], sk[1], x);
        const uint4 qk = quant16<LPV>(x, skale);
        unpack16(sv[0], sv[1], x);
        const uint4 qv = quant16<LPV>(x, svale);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);    // this warp's reads of the stage are done
        if (t < J.n_tok) {
            int64_t row;
            if (J.head_mode) {
                row = J.dst_row0 + t;
            } else {
                // ring slot of the token's frame: first_slot + f < 2 C (f < min(frames, C) -- the job
                // writes at most C frames), so one conditional subtraction replaces the modulo
                const int f = (int)fdiv((uint32_t)t, a.div_frame);
                int slot;
                if (J.use_slots) {
                    slot = J.slots[f];
                } else {
                    slot = J.first_slot + f;
                    if (slot >= Cf) slot -= Cf;
                }
                row = (int64_t)slot * T + (t - f * T);
            }
            const int64_t di = (int64_t)h * J.rows_per_head + row;
            *reinterpret_cast<uint4 *>(J.k8 + di * D + sub * 16) = qk;
            *reinterpret_cast<uint4 *>(J.v8 + di * D + sub * 16) = qv;
            if (sub == 0) {
                J.ks[di] = skale;
                J.vs[di] = svale;
            }
        }
    }
}

struct DequantArgs {
    const int8_t *k8, *v8;
    const float *ks, *vs;
    HistView hv;
    int64_t n_tok;
    int32_t heads;
    float *k_out, *v_out;
};

template <int D>
__global__ void __launch_bounds__(256) dequant_kernel(DequantArgs a) {
    // one thread per (token, head, 16 channels)
    constexpr int CPT = 16;
    const int64_t n = a.n_tok * a.heads * (D / CPT);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int c0 = (int)(i % (D / CPT)) * CPT;
        const int64_t th = i / (D / CPT);
        const int h = (int)(th % a.heads);
        const int64_t t = th / a.heads;
        const int64_t r = (int64_t)h * a.hv.ring_tokens + hist_row(a.hv, t);
        const float sk = a.ks[r], sv = a.vs[r];
        const int8_t *pk = a.k8 + r * D + c0;
        const int8_t *pv = a.v8 + r * D + c0;
        float *ok = a.k_out + (t * a.heads + h) * D + c0;
        float *ov = a.v_out + (t * a.heads + h) * D + c0;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            ok[c] = (float)pk[c] * sk;
            ov[c] = (float)pv[c] * sv;
        }
    }
}

// Tensor map over a job's bf16 K (or V): channels innermost, then heads and tokens in order of
// increasing stride (tokens outermost for [tokens][heads][D] inputs).  The box is D channels of one
// head and TC tokens, which lands in shared memory as [TC][D] either way.
static bool source_map(CUtensorMap *m, const void *base, int64_t n_tok, int heads, int D, int64_t tok_stride,
                       int64_t head_stride, bool tok_outer) {
    const int tc = D == 128 ? AppendCfg<128>::TC : AppendCfg<64>::TC;
    const cuuint64_t nt = (cuuint64_t)(n_tok > 0 ? n_tok : 1);
    const cuuint64_t dims[3] = {(cuuint64_t)D, tok_outer ? (cuuint64_t)heads : nt, tok_outer ? nt : (cuuint64_t)heads};
    const cuuint64_t strides[2] = {(cuuint64_t)(tok_outer ? head_stride : tok_stride) * 2,
                                   (cuuint64_t)(tok_outer ? tok_stride : head_stride) * 2};
    const cuuint32_t box[3] = {(cuuint32_t)D, tok_outer ? 1u : (cuuint32_t)tc, tok_outer ? (cuuint32_t)tc : 1u};
    return make_tensor_map_3d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int D>
static int launch_append(const CUtensorMap *maps, const AppendParams &a, cudaStream_t st) {
    using C = AppendCfg<D>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
        attr = cudaFuncSetAttribute(quant_append_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    });
    if (attr != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(append smem)", (int)attr, cudaGetErrorString(attr));
    const int64_t total = a.job[0].n_chunks + a.job[1].n_chunks;
    if (total >= ((int64_t)1 << 31)) return NOMAS_EINVAL;   // chunk ids are 32-bit
    int64_t blocks = (int64_t)sm_count() * 4;
    if (blocks > total) blocks = total;
    quant_append_kernel<D><<<(unsigned)blocks, kAppendThreads, C::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], a);
    return check_launch("quant_append_kernel launch");
}

}  // namespace nomas

using namespace nomas;

extern "C" int nomas_kv_append(nomas_kv_cache *c, const void *k, const void *v, int64_t tok_stride,
                               int64_t head_stride, int32_t n_frames, const void *head_k, const void *head_v,
                               int32_t head_len, nomas_stream stream) {
    if (!c) return NOMAS_EINVAL;
    const auto &d = c->d;
    if (n_frames < 0 || head_len < 0) return NOMAS_EINVAL;
    if (n_frames == 0 && head_len == 0) return NOMAS_EINVAL;
    if (tok_stride <= 0 || head_stride <= 0 || tok_stride % 8 || head_stride % 8) return NOMAS_EINVAL;
    if (head_stride < d.head_dim && tok_stride < d.head_dim) return NOMAS_EINVAL;
    if (n_frames > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return NOMAS_EINVAL;
    if (head_len > 0 && (!head_k || !head_v || !aligned16(head_k) || !aligned16(head_v))) return NOMAS_EINVAL;
    if (c->head_used + head_len > d.head_store_tokens) return NOMAS_ECAPACITY;
    if (d.window_frames == 0 && c->frames_appended + n_frames > d.capacity_frames) return NOMAS_ECAPACITY;

    const int64_t T = d.tokens_per_frame;
    const int32_t keep = d.window_frames > 0 ? (n_frames < d.window_frames ? n_frames : d.window_frames) : n_frames;
    const int32_t f0 = n_frames - keep;
    const int64_t g0 = c->frames_appended + f0;
    // Retained list after the append: the old frames that still fit the window, then the new ones.  A
    // new frame g takes slot g mod C unless a kept frame holds it (possible only after a selection),
    // in which case it takes the lowest free slot.
    const int64_t Cf = d.capacity_frames;
    size_t n_old = c->ret_frame.size();
    if (d.window_frames > 0) {
        const int64_t room = (int64_t)d.window_frames - keep;
        if ((int64_t)n_old > room) n_old = (size_t)(room > 0 ? room : 0);
    }
    std::vector<int64_t> nf(c->ret_frame.end() - n_old, c->ret_frame.end());
    std::vector<int32_t> ns(c->ret_slot.end() - n_old, c->ret_slot.end());
    std::vector<char> used((size_t)Cf, 0);
    for (int32_t sl : ns) used[sl] = 1;
    std::vector<int32_t> new_slots((size_t)keep);
    bool consecutive = true;
    for (int32_t f = 0; f < keep; ++f) {
        int32_t sl = (int32_t)((g0 + f) % Cf);
        if (used[sl]) {
            sl = 0;
            while (used[sl]) ++sl;   // a free slot exists: kept + new frames <= W <= C
        }
        used[sl] = 1;
        new_slots[f] = sl;
        consecutive = consecutive && sl == (int32_t)((g0 + f) % Cf);
        nf.push_back(g0 + f);
        ns.push_back(sl);
    }
    if (!consecutive && keep > NOMAS_MAX_SELECT_FRAMES) return NOMAS_EUNSUPPORTED;   // not reachable
    const int64_t tc = d.head_dim == 128 ? AppendCfg<128>::TC : AppendCfg<64>::TC;
    if ((int64_t)keep * T >= ((int64_t)1 << 31) || head_len >= ((int64_t)1 << 31)) return NOMAS_EINVAL;

    // both jobs are validated and their maps encoded before the one launch, so a failing call enqueues
    // nothing and leaves the cache as it was
    if (bind_device(c)) return NOMAS_ECUDA;
    AppendParams a{};
    a.heads = d.heads;
    a.tokens_per_frame = d.tokens_per_frame;
    a.capacity_frames = d.capacity_frames;
    a.err = static_cast<int *>(c->buf[NOMAS_BUF_ERR]);
    a.timeout_ns = wait_limit_ns();
    a.div_heads = make_fastdiv((uint32_t)d.heads);
    a.div_frame = make_fastdiv((uint32_t)d.tokens_per_frame);
    CUtensorMap maps[4];
    const void *kv_src[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};
    AppendJob &jv = a.job[0];
    jv.n_tok = (int64_t)keep * T;
    jv.n_chunks = (jv.n_tok + tc - 1) / tc * d.heads;
    jv.head_mode = 0;
    jv.first_slot = (int32_t)(g0 % d.capacity_frames);
    jv.use_slots = consecutive ? 0 : 1;
    for (int32_t f = 0; !consecutive && f < keep; ++f) jv.slots[f] = new_slots[f];
    jv.rows_per_head = (int64_t)d.capacity_frames * T;
    jv.k8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_K8]);
    jv.v8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_V8]);
    jv.ks = static_cast<float *>(c->buf[NOMAS_BUF_KS]);
    jv.vs = static_cast<float *>(c->buf[NOMAS_BUF_VS]);
    if (keep > 0) {
        kv_src[0][0] = static_cast<const __nv_bfloat16 *>(k) + (int64_t)f0 * T * tok_stride;
        kv_src[0][1] = static_cast<const __nv_bfloat16 *>(v) + (int64_t)f0 * T * tok_stride;
    }
    AppendJob &jh = a.job[1];
    jh.n_tok = head_len;
    jh.n_chunks = (jh.n_tok + tc - 1) / tc * d.heads;
    jh.head_mode = 1;
    jh.dst_row0 = c->head_used;
    jh.rows_per_head = d.head_store_tokens;
    jh.k8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_HK8]);
    jh.v8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_HV8]);
    jh.ks = static_cast<float *>(c->buf[NOMAS_BUF_HKS]);
    jh.vs = static_cast<float *>(c->buf[NOMAS_BUF_HVS]);
    if (head_len > 0) {
        kv_src[1][0] = head_k;
        kv_src[1][1] = head_v;
    }
    const bool tok_outer = tok_stride >= head_stride;
    for (int j = 0; j < 2; ++j) {
        a.job[j].tok_outer = tok_outer ? 1 : 0;
        for (int kv = 0; kv < 2; ++kv) {
            // a job without tokens gets a one-token map over its sibling's memory that no chunk reads
            const void *base = kv_src[j][kv] ? kv_src[j][kv] : kv_src[j ^ 1][kv];
            if (!source_map(&maps[2 * j + kv], base, a.job[j].n_tok, d.heads, d.head_dim, tok_stride, head_stride,
                            tok_outer))
                return NOMAS_ECUDA;
        }
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int rc = d.head_dim == 128 ? launch_append<128>(maps, a, st) : launch_append<64>(maps, a, st);
    if (rc) return rc;
    c->frames_appended += n_frames;
    c->head_used += head_len;
    c->segments += 1;
    c->version += 1;
    c->ret_frame.swap(nf);
    c->ret_slot.swap(ns);
    return NOMAS_OK;
}

extern "C" int nomas_kv_dequant(const nomas_kv_cache *c, float *k_out, float *v_out, nomas_stream stream) {
    if (!c) return NOMAS_EINVAL;
    const HistView hv = hist_view(c);
    if (hv.tokens == 0) return NOMAS_OK;
    if (!k_out || !v_out || !aligned16(k_out) || !aligned16(v_out)) return NOMAS_EINVAL;
    if (bind_device(c)) return NOMAS_ECUDA;
    DequantArgs a{};
    a.k8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_K8]);
    a.v8 = static_cast<const int8_t *>(c->buf[NOMAS_BUF_V8]);
    a.ks = static_cast<const float *>(c->buf[NOMAS_BUF_KS]);
    a.vs = static_cast<const float *>(c->buf[NOMAS_BUF_VS]);
    a.hv = hv;
    a.n_tok = hv.tokens;
    a.heads = c->d.heads;
    a.k_out = k_out;
    a.v_out = v_out;
    const int64_t n = hv.tokens * c->d.heads * (c->d.head_dim / 16);
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (c->d.head_dim == 128) dequant_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(a);
    else dequant_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(a);
    return check_launch("dequant_kernel launch");
}
