// nomas_kv_append / nomas_kv_dequant: INT8 quantise-append of a finished segment's K/V into the
// sliding-window ring (fluxbbs.com "单卡 4090 怎么做到的", first and second techniques: INT8
// storage with float scales; 18 retained history latent frames) and the description-head store.
//
// HBM-bound: per (token, head) 2*D bf16 read, 2*D int8 + 2 fp32 written.  One group of D/8 lanes
// handles one (token, head): each lane holds 8 channels of K and 8 of V in one 16-byte load each,
// the absmax is reduced with xor-shuffles inside the group, and each lane stores 8 codes (8 bytes).
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

// rint(x / s) in fp32 with IEEE division and round-half-even, clamped to [-127, 127].
// y = x * RN(1/s) is within 2^-16 + 2^-17 of RN(x/s) for |x/s| <= 127 (two roundings of relative
// size 2^-24 each, one more for RN(x/s) itself), so when y is farther than 2^-15 from the nearest
// half-integer both round to the same integer; otherwise (rare) the exact quotient is computed.
__device__ __forceinline__ float quant_code(float x, float s, float r) {
    const float y = x * r;
    const float fl = floorf(y);
    const float dist = fabsf((y - fl) - 0.5f);
    float q = (dist > 0x1p-15f) ? rintf(y) : rintf(__fdiv_rn(x, s));
    return fminf(fmaxf(q, -127.0f), 127.0f);
}

template <int LPV>
__device__ __forceinline__ float group_max(float a) {
#pragma unroll
    for (int off = LPV / 2; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    return a;
}

__device__ __forceinline__ void unpack8(const uint4 &w, float (&x)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(u[i] << 16);
        x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

template <int LPV>
__device__ __forceinline__ uint2 quant8(const float (&x)[8], float &s_out) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(x[i]));
    a = group_max<LPV>(a);
    const float s = __fdiv_rn(a, 127.0f);
    s_out = s;
    uint32_t lo = 0, hi = 0;
    if (s > 0.0f) {
        const float r = __frcp_rn(s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t b = (uint32_t)((int)quant_code(x[i], s, r)) & 0xFFu;
            if (i < 4) lo |= b << (8 * i);
            else hi |= b << (8 * (i - 4));
        }
    }
    return make_uint2(lo, hi);
}

template <int D>
__global__ void __launch_bounds__(256) quant_append_kernel(AppendArgs a) {
    constexpr int LPV = D / 8;          // lanes per (token, head) vector
    constexpr int GPW = 32 / LPV;       // groups per warp
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPV;
    const int grp = lane / LPV;
    const int64_t n_items = a.n_tok * a.heads;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t wstride = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp0 * GPW; base < n_items; base += wstride * GPW) {
        const int64_t it = base + grp;
        const bool ok = it < n_items;
        const int64_t itc = ok ? it : base;
        // item order: head-major, so consecutive groups write consecutive destination rows
        const int h = (int)(itc / a.n_tok);
        const int64_t t = itc - (int64_t)h * a.n_tok;
        const int64_t src = t * a.tok_stride + (int64_t)h * a.head_stride + sub * 8;
        const uint4 rk = __ldg(reinterpret_cast<const uint4 *>(a.k + src));
        const uint4 rv = __ldg(reinterpret_cast<const uint4 *>(a.v + src));
        float xk[8], xv[8];
        unpack8(rk, xk);
        unpack8(rv, xv);
        float sk, sv;
        const uint2 qk = quant8<LPV>(xk, sk);
        const uint2 qv = quant8<LPV>(xv, sv);
        int64_t row;
        if (a.head_mode) {
            row = a.dst_row0 + t;
        } else {
            const int64_t f = t / a.tokens_per_frame;
            const int64_t slot = (a.first_slot + f) % a.capacity_frames;
            row = slot * a.tokens_per_frame + (t - f * a.tokens_per_frame);
        }
        const int64_t di = (int64_t)h * a.rows_per_head + row;
        if (ok) {
            *reinterpret_cast<uint2 *>(a.k8 + di * D + sub * 8) = qk;
            *reinterpret_cast<uint2 *>(a.v8 + di * D + sub * 8) = qv;
            if (sub == 0) {
                a.ks[di] = sk;
                a.vs[di] = sv;
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
    const int64_t groups = a.n_tok * a.heads;
    const int64_t threads = groups * (D / 8);
    int64_t blocks = (threads + 255) / 256;
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
