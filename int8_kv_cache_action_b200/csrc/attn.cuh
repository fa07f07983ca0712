// Parameters and device helpers shared by the two attention kernels: attn_fwd_kernel (one 128-row query
// block per CTA, attn.cu) and attn_pair_kernel (the two query blocks of a tile list per CTA,
// attn_pair.cu).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace nomas {

constexpr float kRescaleThreshold = 6.0f;   // log2 units: P <= 64

struct AttnParams {
    const float *ksl, *vsl;     // retained-history scales in age order, [H][hist_stride]
    const float *hks, *hvs;     // description-head scales, [H][head_rows]
    int64_t hist_stride, head_rows;
    // mask buffer
    const uint8_t *mask;
    const int4 *lists;
    const int32_t *counts;
    const int2 *txtwin;         // per text token: frame window (tails) or [0, kAlwaysHi) (head)
    MaskHeader expect;
    const WsHeader *ws_hdr;     // written by nomas_attn_prepare
    WsHeader ws_expect;
    int32_t sparse;
    int32_t text_rows;          // query rows are the current text (NOMAS_MODE_TEXT), else the video
    int32_t head_len;           // description-head tokens at the front of the current text
    int32_t n_pairs;
    // queries and shapes
    const __nv_bfloat16 *q;
    int64_t tok_stride, head_stride;
    int32_t H, T;
    FastDiv divT;               // token -> frame (every token index here is below 2^31)
    int64_t Nq;
    float scale_log2;           // softmax_scale * log2(e)
    float *out;
    float *lse;
    int *err;
    uint64_t timeout_ns;
    // text query rows: each list cut into shares of share_len entries, share blockIdx.z per CTA, which
    // writes its O without normalisation and (offset, row sum) per row for attn_combine_kernel;
    // share_len == 0: the whole list, normalised output
    int32_t share_len;
    float *part_o;              // [share][Nq][H][D]
    float2 *part_ml;            // [share][H][Nq]
    // dense calls of the pair kernel (grid x = work units, unit = head * n_pairs + pair): units
    // [0, n_full) run whole lists; each of the n_tail units after them runs as tail_shares CTAs of
    // tail_len entries that write unnormalised partials for attn_combine_tail_kernel, so that the
    // partial last wave of whole lists becomes one wave of short shares (tail_len == 0: no split)
    int32_t n_full, n_tail, tail_shares, tail_len;
    float *tail_o;              // [tail_shares][n_tail][2 * 128 rows][D]
    float2 *tail_ml;            // [tail_shares][n_tail][2 * 128 rows]
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x for x <= 6 on the FMA pipe (the MUFU unit's exponential throughput equals the tensor pipe's
// rate per score at head_dim 128, so part of the exponentials are taken off it): x is clamped at -125,
// n = rint(x) by the 1.5 * 2^23 add, f = x - n lies in [-1/2, 1/2], 2^f comes from a degree-3
// polynomial fitted by weighted least squares to the relative error on Chebyshev nodes (maximum
// relative error 7.5e-5, below fp16's half unit in the last place, 2^-12), and n is added to the
// exponent field.
__device__ __forceinline__ float2 exp2_poly(float2 x) {
    x.x = fmaxf(x.x, -125.0f);
    x.y = fmaxf(x.y, -125.0f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
    const float2 n = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
    const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
    float2 q = __ffma2_rn(make_float2(0.055171605f, 0.055171605f), f, make_float2(0.24261111f, 0.24261111f));
    q = __ffma2_rn(q, f, make_float2(0.69326097f, 0.69326097f));
    q = __ffma2_rn(q, f, make_float2(0.99992806f, 0.99992806f));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

#ifndef NOMAS_POLY_PAIRS
#define NOMAS_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = NOMAS_POLY_PAIRS;   // of every 16 column pairs, this many take exp2_poly

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ bool is_cached(int kind) { return kind == kKindHist || kind == kKindPriorHead; }

// Walks a CTA's tile list, each entry loaded two entries ahead of its use.
struct ListCursor {
    const int4 *list;
    int n, j;
    int4 a, b;
    __device__ __forceinline__ ListCursor(const int4 *l, int n_) : list(l), n(n_), j(0) {
        a = n > 0 ? list[0] : make_int4(0, 0, 0, 0);
        b = n > 1 ? list[1] : make_int4(0, 0, 0, 0);
    }
    // the next entry carrying `bit`; false at the end of the list
    __device__ __forceinline__ bool next(int bit, int4 &e) {
        while (j < n) {
            const int4 c = a;
            a = b;
            b = (j + 2 < n) ? list[j + 2] : make_int4(0, 0, 0, 0);
            ++j;
            if (c.x & bit) {
                e = c;
                return true;
            }
        }
        return false;
    }
};

// Column `col` of a tile-list entry: the raw key and value scales of a cached key (1 and 0 for a key
// of bf16 source; 0 and 0 past the tile's valid keys) and, when the tile is masked for some query block
// of the CTA, the key's visibility code (never read otherwise).
struct ColInfo {
    float ks, vs;
    VisCode w;
    bool masked;
};
__device__ __forceinline__ ColInfo column_info(const AttnParams &p, int h, const int4 &e, int col, bool masked) {
    ColInfo ci{0.0f, 0.0f, key_none(), masked};
    const int kind = e.x & 3;
    const int64_t start = e.y;
    if (col < e.z) {
        if (!masked) {
            // codes unused: the whole tile is visible to every row
        } else if (kind == kKindText) {
            if (start + col < p.head_len) {
                ci.w = key_always();
            } else {
                const int2 w = p.txtwin[start + col];
                ci.w = key_tail(w.x, w.y);
            }
        } else if (kind == kKindCur) {
            ci.w = key_video((int)fdiv((uint32_t)(start + col), p.divT));
        } else {
            ci.w = key_always();
        }
        if (is_cached(kind)) {
            const bool hist = kind == kKindHist;
            const int64_t i = (int64_t)h * (hist ? p.hist_stride : p.head_rows) + start + col;
            ci.ks = __ldg((hist ? p.ksl : p.hks) + i);
            ci.vs = __ldg((hist ? p.vsl : p.hvs) + i);
        } else {
            ci.ks = 1.0f;
        }
    }
    return ci;
}

// Softmax merge of one (row, head) over list shares: with M the largest offset among the shares that saw
// a visible key, O = sum_s O_s 2^(m_s - M) / sum_s l_s 2^(m_s - M) and lse = (M + log2 of the
// denominator) ln 2 (the kernels' log2 domain).  One warp, D / 32 channels per lane; share s of the
// row's partial output starts at o + s * o_stride, its (offset, row sum) at ml[s * ml_stride].
template <int D>
__device__ __forceinline__ void merge_shares(const float *o, int64_t o_stride, const float2 *ml, int64_t ml_stride,
                                             int n_share, float *dst, float *lse, int lane) {
    float M = -INFINITY;
    for (int s = 0; s < n_share; ++s) {
        const float2 v = ml[s * ml_stride];
        if (v.y > 0.0f) M = fmaxf(M, v.x);
    }
    constexpr int PL = D / 32;
    float acc[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) acc[i] = 0.0f;
    float L = 0.0f;
    for (int s = 0; s < n_share; ++s) {
        const float2 v = ml[s * ml_stride];
        if (!(v.y > 0.0f)) continue;
        const float wgt = exp2f(v.x - M);
        L += v.y * wgt;
        const float *src = o + s * o_stride;
#pragma unroll
        for (int i = 0; i < PL; ++i) acc[i] += src[lane + 32 * i] * wgt;
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int i = 0; i < PL; ++i) dst[lane + 32 * i] = acc[i] * inv;
    if (lse && lane == 0) *lse = (M + log2f(L)) * 0.69314718055994530942f;
}

// The pair kernel (head_dim 128): grid (work units, 1, list shares); with a tail split, grid x =
// n_full + n_tail * tail_shares.
int launch_attn_pair(const AttnParams &p, dim3 grid, const CUtensorMap *maps, cudaStream_t st);
// Merge of the tail shares of a pair-kernel call into out / lse.
int launch_combine_tail(const AttnParams &p, int D, cudaStream_t st);

}  // namespace nomas
