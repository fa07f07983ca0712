// Pre-pass of nomas_attn_fwd: the attention kernel's operand copies (see prep.cuh).
#include "prep.cuh"

namespace nomas {

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
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

// bf16 [n][H][D] (token / head strides in elements) -> fp16 [H][n][D], for up to two tensors.  One
// block converts 64 tokens x D of one head (a contiguous 64 x D run of the destination).
__device__ __forceinline__ void keys_f16_block(const F16Jobs &jobs, const uint3 blk) {
    if (blk.x == 0 && blk.y == 0 && blk.z == 0 && threadIdx.x == 0) *jobs.hdr_dst = jobs.hdr;
    const F16Job J = blk.z ? jobs.job[1] : jobs.job[0];
    const int h = blk.y;
    const int64_t t0 = (int64_t)blk.x * 64;
    if (t0 >= J.n) return;
    const int cpr = jobs.D / 8;   // 16-byte chunks per row
    const int rows = J.n - t0 < 64 ? (int)(J.n - t0) : 64;
    const uint4 *src = reinterpret_cast<const uint4 *>(J.src + t0 * jobs.tok_stride + (int64_t)h * jobs.head_stride);
    uint4 *dst = reinterpret_cast<uint4 *>(J.dst + ((int64_t)h * J.n + t0) * jobs.D);
    const int64_t srow = jobs.tok_stride / 8;   // source row stride in 16-byte chunks
    bool bad = false;
    for (int i = threadIdx.x; i < rows * cpr; i += blockDim.x) {
        const int r = i / cpr, c = i - r * cpr;
        const uint4 h = bf16x8_to_f16(__ldg(src + r * srow + c));
        bad |= f16x8_nonfinite(h);
        dst[i] = h;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_device_error(jobs.err, NOMAS_ERANGE, 30);
}

// bf16 [n][H][D] -> fp16 V^T [H][D][np] (np = n rounded up to 8; the padding is zero), for up to
// two tensors.  One block transposes 64 tokens x D of one head through shared memory, held as 32-bit
// words (two adjacent channels) with token t's word w stored at column w ^ 4 (t / 8): the 16-byte
// row writes stay contiguous, and a warp reading one word of 8 tokens spaced 8 apart for 4
// adjacent words hits 32 distinct banks.  Each thread then emits 8 tokens of two channel rows.

__device__ __forceinline__ void values_t16_block(const VtJobs &jobs, const uint3 blk, uint32_t *tile) {
    // tile: [token][word] (64 x 64 words), D / 2 words per token used
    const VtJob J = blk.z ? jobs.job[1] : jobs.job[0];
    const int h = blk.y;
    const int64_t t0 = (int64_t)blk.x * 64;
    if (t0 >= J.np) return;
    const int D = jobs.D;
    const int W = D / 2;                  // words per token row
    const int cpr = D / 8;                // 16-byte chunks per token row
    bool bad = false;
    for (int i = threadIdx.x; i < 64 * cpr; i += blockDim.x) {
        const int r = i / cpr, k = i % cpr;
        const int64_t t = t0 + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < J.n)
            v = bf16x8_to_f16(__ldg(reinterpret_cast<const uint4 *>(J.src + t * jobs.tok_stride +
                                                                    (int64_t)h * jobs.head_stride) + k));
        bad |= f16x8_nonfinite(v);
        *reinterpret_cast<uint4 *>(&tile[r * W + ((4 * k) ^ ((r >> 3) << 2))]) = v;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_device_error(jobs.err, NOMAS_ERANGE, 31);
    for (int i = threadIdx.x; i < W * 8; i += blockDim.x) {
        const int w = (i >> 5) * 4 + (i & 3);   // word: channels 2w, 2w + 1
        const int c = (i >> 2) & 7;             // tokens [t0 + 8c, t0 + 8c + 8)
        const int64_t t = t0 + c * 8;
        if (t >= J.np) continue;
        uint32_t x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = tile[(c * 8 + j) * W + (w ^ (c << 2))];
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            lo[k] = __byte_perm(x[2 * k], x[2 * k + 1], 0x5410);   // channel 2w of tokens 2k, 2k + 1
            hi[k] = __byte_perm(x[2 * k], x[2 * k + 1], 0x7632);   // channel 2w + 1
        }
        __half *d0 = J.dst + ((int64_t)h * D + 2 * w) * J.np + t;
        *reinterpret_cast<uint4 *>(d0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4 *>(d0 + J.np) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
}

// INT8 codes of the cache as exact fp16 integers, in the layouts of the attention kernel's TMA boxes:
//   z = 0: ring rows of the retained history in age order -> keys [H][Lh][D], V^T [H][D][lhp] (lhp =
//          Lh rounded up to 16, zero padding), key / value scales [H][lhp];
//   z = 1: description-head store rows [0, Lp) -> keys [H][Lp][D], V^T [H][D][lpp] (its scales are
//          read in place).
// One block converts 64 tokens x D of one head; values are transposed through shared memory.

__device__ __forceinline__ void hist_prep_block(const HistPrep &P, const uint3 blk, int8_t (*tile)[128 + 16]) {
    const bool heads = blk.z == 1;
    const int h = blk.y;
    const int64_t n = heads ? P.Lp : P.Lh, np = heads ? P.lpp : P.lhp;
    const int64_t t0 = (int64_t)blk.x * 64;
    if (t0 >= np) return;
    const int D = P.D;
    const int cpr = D / 16;
    const int8_t *ksrc = heads ? P.hk8 : P.k8, *vsrc = heads ? P.hv8 : P.v8;
    __half *kdst = heads ? P.kp : P.kh;
    auto src_row = [&](int64_t a) -> int64_t {
        return heads ? (int64_t)h * P.head_rows + a : (int64_t)h * P.hv.ring_tokens + hist_row(P.hv, a);
    };
    for (int i = threadIdx.x; i < 64 * cpr; i += blockDim.x) {
        const int r = i / cpr, c = i % cpr;
        const int64_t a = t0 + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (a < n) {
            const int64_t sr = src_row(a);
            v = __ldg(reinterpret_cast<const uint4 *>(vsrc + sr * D) + c);
            uint4 lo, hi;
            i8x16_to_f16(__ldg(reinterpret_cast<const uint4 *>(ksrc + sr * D) + c), lo, hi);
            uint4 *kd = reinterpret_cast<uint4 *>(kdst + ((int64_t)h * n + a) * D) + 2 * c;
            kd[0] = lo;
            kd[1] = hi;
        }
        *reinterpret_cast<uint4 *>(&tile[r][c * 16]) = v;
    }
    // scales: the history's are copied in age order; every cached value scale must keep
    // 64 * scale within fp16 and every key scale must be finite (checked for the heads too)
    bool bad = false;
    if (threadIdx.x < 64) {
        const int64_t a = t0 + threadIdx.x;
        if (a < np) {
            float ks = 0.0f, vs = 0.0f;
            if (a < n) {
                const int64_t sr = src_row(a);
                ks = __ldg((heads ? P.hks : P.ks) + sr);
                vs = __ldg((heads ? P.hvs : P.vs) + sr);
                bad = !(vs <= kMaxValueScale) || !(fabsf(ks) <= 3.4028235e38f);
            }
            if (!heads) {
                P.ksl[(int64_t)h * P.lhp + a] = ks;
                P.vsl[(int64_t)h * P.lhp + a] = vs;
            }
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_device_error(P.err, NOMAS_ERANGE, 32);
    __half *dst = heads ? P.vpt : P.vht;
    for (int i = threadIdx.x; i < D * 4; i += blockDim.x) {
        const int d = i / 4, c = i % 4;   // row d, tokens [t0 + 16c, t0 + 16c + 16)
        const int64_t t = t0 + c * 16;
        if (t >= np) continue;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = (uint32_t)(uint8_t)tile[c * 16 + 4 * k][d] | ((uint32_t)(uint8_t)tile[c * 16 + 4 * k + 1][d] << 8) |
                   ((uint32_t)(uint8_t)tile[c * 16 + 4 * k + 2][d] << 16) |
                   ((uint32_t)(uint8_t)tile[c * 16 + 4 * k + 3][d] << 24);
        uint4 lo, hi;
        i8x16_to_f16(make_uint4(w[0], w[1], w[2], w[3]), lo, hi);
        uint4 *vd = reinterpret_cast<uint4 *>(dst + ((int64_t)h * D + d) * np + t);
        vd[0] = lo;
        vd[1] = hi;
    }
}

// The three copies of a call in one launch: blocks [0, n_k) convert keys, [n_k, n_k + n_v) transpose
// values, the rest widen the history and the description heads; every block is independent, so the
// block scheduler interleaves them and no copy waits for another's tail.
struct PrepGrid {
    dim3 k, v, h;       // the grid of each part (zero blocks: part absent)
    uint32_t n_k, n_v;  // blocks of the first two parts
};

__device__ __forceinline__ uint3 block_of(uint32_t b, const dim3 &g) {
    return make_uint3(b % g.x, (b / g.x) % g.y, b / (g.x * g.y));
}

__global__ void __launch_bounds__(256) prepare_kernel(const F16Jobs fj, const VtJobs vj, const HistPrep hp,
                                                      const PrepGrid g) {
    __shared__ __align__(16) uint32_t smem[64 * 64];   // the value transpose tile or the history tile
    const uint32_t b = blockIdx.x;
    if (b < g.n_k) {
        keys_f16_block(fj, block_of(b, g.k));
    } else if (b < g.n_k + g.n_v) {
        values_t16_block(vj, block_of(b - g.n_k, g.v), smem);
    } else {
        static_assert(64 * (128 + 16) <= 64 * 64 * 4, "the history tile fits");
        hist_prep_block(hp, block_of(b - g.n_k - g.n_v, g.h), reinterpret_cast<int8_t (*)[128 + 16]>(smem));
    }
}

int launch_prepare(const F16Jobs &fj, const VtJobs &vj, bool two, int64_t max_np, const HistPrep *hp, cudaStream_t st) {
    PrepGrid g{};
    int64_t nmax = 0;
    for (int j = 0; j < fj.n_jobs; ++j) nmax = fj.job[j].n > nmax ? fj.job[j].n : nmax;
    g.k = dim3((unsigned)((nmax + 63) / 64), (unsigned)fj.H, (unsigned)fj.n_jobs);
    g.v = dim3((unsigned)((max_np + 63) / 64), (unsigned)vj.H, two ? 2u : 1u);
    const int64_t hmax = hp ? (hp->lhp > hp->lpp ? hp->lhp : hp->lpp) : 0;
    g.h = dim3((unsigned)((hmax + 63) / 64), hp ? (unsigned)hp->H : 0u, 2u);
    const int64_t nk = (int64_t)g.k.x * g.k.y * g.k.z, nv = (int64_t)g.v.x * g.v.y * g.v.z;
    const int64_t nh = (int64_t)g.h.x * g.h.y * g.h.z;
    if (nk + nv + nh >= ((int64_t)1 << 31)) return NOMAS_EINVAL;
    g.n_k = (uint32_t)nk;
    g.n_v = (uint32_t)nv;
    if (nk + nv + nh == 0) return NOMAS_OK;
    prepare_kernel<<<(unsigned)(nk + nv + nh), 256, 0, st>>>(fj, vj, hp ? *hp : HistPrep{}, g);
    return check_launch("prepare_kernel launch");
}

}  // namespace nomas
