// nomas_kv_append / nomas_kv_dequant: INT8 quantise-append of a finished segment's K/V into the
// sliding-window ring (fluxbbs.com "单卡 4090 怎么做到的", first and second techniques: INT8
// storage with float scales; 18 retained history latent frames) and the description-head store.
//
// HBM-bound: per (token, head) 2*D bf16 read, 2*D int8 + 2 fp32 written.  One group of D/16 lanes
// handles one (token, head): each lane holds 16 channels of K and 16 of V (two 16-byte loads each),
// the absmax is reduced with xor-shuffles inside the group, and each lane stores 16 codes.
#include "common.cuh"

namespace nomas {

struct AppendArgs {
    const __nv_bfloat16 *k;   // first token to write
    const __nv_bfloat16 *v;
    int64_t tok_stride, head_stride;
    int64_t n_tok;            // tokens to write
    int32_t heads;
    int32_t tokens_per_frame;
    int32_t capacity_frames;
    int32_t first_slot;       // ring slot of the first token's frame (video mode)
    int32_t head_mode;        // 1: destination rows dst_row0 + t (head store)
    int64_t dst_row0;
    int64_t rows_per_head;    // destination rows per head
    int8_t *k8;
    int8_t *v8;
    float *ks;
    float *vs;
};

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

// s = RN(a / 127) for a = absmax of bf16 values, without the division routine: q0 = RN(a c) with
// c = RN(1/127), the remainder a - 127 q0 is exact by FMA, and s = RN(q0 + (a - 127 q0) c) is
// Markstein's correction step ("Computation of elementary functions on the IBM RISC System/6000
// processor", 1990).  Checked by exact rational arithmetic against RN(a / 127) for every bf16 a in
// [2^-110, max finite], where q0 and s are normals and the remainder (a subnormal at the low end) is
// exact; zero gives zero, and subnormal or non-finite a take the IEEE division.
__device__ __forceinline__ float div127(float a) {
    constexpr float c = 0x1.020408p-7f;                   // RN(1/127)
    const float q0 = __fmul_rn(a, c);
    const float s = __fmaf_rn(__fmaf_rn(-q0, 127.0f, a), c, q0);
    if (!(a >= 0x1p-110f && a <= 0x1.fffffep127f) && a != 0.0f) return __fdiv_rn(a, 127.0f);
    return s;
}

// 1/s for normal s: the hardware approximation (PTX rcp.approx.f32, relative error about 2^-23)
// refined by one Newton-Raphson step r = r0 + r0 (1 - s r0), both by FMA, leaves a relative error
// below 2^-24 + 2^-40.
__device__ __forceinline__ float recip_nr(float s) {
    float r0;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r0) : "f"(s));
    return __fmaf_rn(r0, __fmaf_rn(-s, r0, 1.0f), r0);
}

// Codes rint(x / s) in fp32 with IEEE division and round-half-even for the 16 channels this lane
// holds; s = RN(absmax / 127) over the group's D channels, so |x / s| <= 127 (1 + 2^-23) and every
// code lies in [-127, 127].
// y = x * r with r = 1/s to relative 2^-24 + 2^-40 is within 2^-16 + 2^-17 of RN(x/s) for
// |x/s| <= 127 (about 127 * 2^-23 from r and the rounding of y, 2^-18 for RN(x/s) itself), so when y
// is farther than 2^-15 from the nearest half-integer both round to the same integer.  Otherwise
// the exact quotient decides: rarely, and always for s below 2^-125, where r is a NaN.  The warp
// takes that branch only when one of its lanes needs it.
// Rounding uses t = y + 1.5 * 2^23: the fp32 add rounds y half-to-even to an integer and leaves it,
// as a two's-complement byte, in the low byte of t's bit pattern; y - (t - 1.5 * 2^23) is exact.
template <int LPV>
__device__ __forceinline__ uint4 quant16(const float (&x)[16], float &s_out) {
    constexpr float kMagic = 12582912.0f;                 // 1.5 * 2^23
    constexpr float kFar = 0.5f - 0x1p-15f;               // |y - rint(y)| below this: not near a tie
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
    a = group_max<LPV>(a);
    const float s = div127(a);
    s_out = s;
    const bool nz = s > 0.0f;
    const float r = s >= 0x1p-125f ? recip_nr(s) : (nz ? __int_as_float(0x7fffffff) : 0.0f);
    const float2 r2 = make_float2(r, r), m2 = make_float2(kMagic, kMagic), nm2 = make_float2(-kMagic, -kMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    uint32_t tb[16];
    bool slow = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 y = __fmul2_rn(make_float2(x[2 * i], x[2 * i + 1]), r2);
        const float2 t = __fadd2_rn(y, m2);
        const float2 q = __fadd2_rn(t, nm2);
        const float2 d = __ffma2_rn(q, neg1, y);          // y - rint(y), exact
        slow |= !(fabsf(d.x) < kFar) || !(fabsf(d.y) < kFar);   // NaN (tiny s) counts as near
        tb[2 * i] = __float_as_uint(t.x);
        tb[2 * i + 1] = __float_as_uint(t.y);
    }
    if (__any_sync(0xffffffffu, slow && nz)) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float y = x[i] * r;
            const float d = y - __fsub_rn(__fadd_rn(y, kMagic), kMagic);
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

// Work unit of a warp: one head of a block of kTokBlock consecutive tokens, one token per group of
// D/16 lanes (16 channels per lane).  The warp issues all its 16-byte loads before quantising and
// writes kTokBlock consecutive destination rows and scales of that head.  Index arithmetic is one
// 32-bit division per unit; destination rows advance incrementally across frame boundaries.  At most
// 64 registers, so four 256-thread blocks share an SM.
template <int D>
constexpr int kTokBlock = 32 / (D / 16);    // one token per group of D/16 lanes

template <int D>
__global__ void __launch_bounds__(256, 4) quant_append_kernel(AppendArgs a) {
    constexpr int LPV = D / 16;             // lanes per (token, head) vector
    constexpr int GPW = 32 / LPV;           // groups per warp
    constexpr int IPG = kTokBlock<D> / GPW; // tokens per group and unit
    static_assert(IPG >= 1 && IPG * GPW == kTokBlock<D>, "token block split");
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPV;
    const int grp = lane / LPV;
    const int n_tok = (int)a.n_tok;
    const int T = a.tokens_per_frame, C = a.capacity_frames;
    const int n_units = (n_tok + kTokBlock<D> - 1) / kTokBlock<D> * a.heads;
    const int warp0 = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int nwarps = (int)(((int64_t)gridDim.x * blockDim.x) >> 5);
    for (int unit = warp0; unit < n_units; unit += nwarps) {
        const int tb = unit / a.heads;
        const int h = unit - tb * a.heads;
        const int t0 = tb * kTokBlock<D> + grp * IPG;
        uint4 rk[IPG][2], rv[IPG][2];
#pragma unroll
        for (int i = 0; i < IPG; ++i) {
            const int t = t0 + i < n_tok ? t0 + i : 0;   // rows past the end read token 0, dropped below
            const int64_t src = (int64_t)t * a.tok_stride + (int64_t)h * a.head_stride + sub * 16;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                rk[i][c] = __ldg(reinterpret_cast<const uint4 *>(a.k + src) + c);
                rv[i][c] = __ldg(reinterpret_cast<const uint4 *>(a.v + src) + c);
            }
        }
        // destination row of t0: ring slot of its frame (video) or the head store's next row
        int r = 0, slot = 0;
        if (!a.head_mode) {
            const int f = t0 / T;
            r = t0 - f * T;
            slot = (a.first_slot + f) % C;
        }
#pragma unroll
        for (int i = 0; i < IPG; ++i) {
            float x[16];
            float sk, sv;
            unpack16(rk[i][0], rk[i][1], x);
            const uint4 qk = quant16<LPV>(x, sk);
            unpack16(rv[i][0], rv[i][1], x);
            const uint4 qv = quant16<LPV>(x, sv);
            const int64_t row = a.head_mode ? a.dst_row0 + t0 + i : (int64_t)slot * T + r;
            const int64_t di = (int64_t)h * a.rows_per_head + row;
            if (t0 + i < n_tok) {
                *reinterpret_cast<uint4 *>(a.k8 + di * D + sub * 16) = qk;
                *reinterpret_cast<uint4 *>(a.v8 + di * D + sub * 16) = qv;
                if (sub == 0) {
                    a.ks[di] = sk;
                    a.vs[di] = sv;
                }
            }
            if (++r == T) {   // next token starts the next frame
                r = 0;
                slot = slot + 1 == C ? 0 : slot + 1;
            }
        }
    }
}

struct DequantArgs {
    const int8_t *k8, *v8;
    const float *ks, *vs;
    int64_t rows_per_head, ring_tokens, first_tok, n_tok;
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
        const int64_t phys = (a.first_tok + t) % a.ring_tokens;
        const int64_t r = (int64_t)h * a.rows_per_head + phys;
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

static int launch_append(const AppendArgs &a, int D, cudaStream_t st) {
    if (a.n_tok <= 0) return NOMAS_OK;
    if (a.n_tok >= (int64_t)1 << 30) return NOMAS_EINVAL;   // 32-bit token indices
    const int64_t tbk = D == 128 ? kTokBlock<128> : kTokBlock<64>;
    const int64_t units = (a.n_tok + tbk - 1) / tbk * a.heads;   // one warp each
    if (units >= (int64_t)1 << 31) return NOMAS_EINVAL;
    int64_t blocks = (units * 32 + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (D == 128) quant_append_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(a);
    else quant_append_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(a);
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

    if (bind_device(c)) return NOMAS_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t T = d.tokens_per_frame;
    const int32_t keep = d.window_frames > 0 ? (n_frames < d.window_frames ? n_frames : d.window_frames) : n_frames;
    const int32_t f0 = n_frames - keep;
    const int64_t g0 = c->frames_appended + f0;

    AppendArgs a{};
    a.tok_stride = tok_stride;
    a.head_stride = head_stride;
    a.heads = d.heads;
    a.tokens_per_frame = d.tokens_per_frame;
    a.capacity_frames = d.capacity_frames;
    int rc = NOMAS_OK;
    if (keep > 0) {
        a.k = static_cast<const __nv_bfloat16 *>(k) + (int64_t)f0 * T * tok_stride;
        a.v = static_cast<const __nv_bfloat16 *>(v) + (int64_t)f0 * T * tok_stride;
        a.n_tok = (int64_t)keep * T;
        a.first_slot = (int32_t)(g0 % d.capacity_frames);
        a.head_mode = 0;
        a.rows_per_head = (int64_t)d.capacity_frames * T;
        a.k8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_K8]);
        a.v8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_V8]);
        a.ks = static_cast<float *>(c->buf[NOMAS_BUF_KS]);
        a.vs = static_cast<float *>(c->buf[NOMAS_BUF_VS]);
        rc = launch_append(a, d.head_dim, st);
        if (rc) return rc;
    }
    if (head_len > 0) {
        a.k = static_cast<const __nv_bfloat16 *>(head_k);
        a.v = static_cast<const __nv_bfloat16 *>(head_v);
        a.n_tok = head_len;
        a.first_slot = 0;
        a.head_mode = 1;
        a.dst_row0 = c->head_used;
        a.rows_per_head = d.head_store_tokens;
        a.k8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_HK8]);
        a.v8 = static_cast<int8_t *>(c->buf[NOMAS_BUF_HV8]);
        a.ks = static_cast<float *>(c->buf[NOMAS_BUF_HKS]);
        a.vs = static_cast<float *>(c->buf[NOMAS_BUF_HVS]);
        rc = launch_append(a, d.head_dim, st);
        if (rc) return rc;
    }
    c->frames_appended += n_frames;
    c->head_used += head_len;
    c->segments += 1;
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
    a.rows_per_head = hv.ring_tokens;
    a.ring_tokens = hv.ring_tokens;
    a.first_tok = hv.first_tok;
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
