// INT8-weight / BF16-compute linear layer of the DiT (fluxbbs.com "单卡 4090 怎么做到的", first
// technique: weights stored as INT8 with float scale factors, dequantised back to BF16 at compute
// time; the linear layers compute in BF16).  The reading (per-output-row scales, bf16-rounded
// dequantised weights, fp32 accumulation) is stated in nomas.h.
//
// Kernels:
//   w8_quantize_kernel   one CTA per weight row: absmax, s = RN(absmax / 127), codes
//   w8_dequant_kernel    bf16(RN(code * s)), 16 weights per thread (HBM-bound)
//   gemm2_bf16_kernel    y = x W^T on the tensor cores (more than 128 rows): persistent clusters of two
//                        CTAs on an SM pair, tiles of 256 x 256 computed by tcgen05.mma.cta_group::2
//                        M256 N256 K16 from the even CTA; each CTA stages 128 rows of A and 128 rows
//                        of B per K step of 64 through a six-stage TMA ring (16 + 16 KB, 128-byte
//                        swizzle, no multicast) and holds its 128 accumulator rows in TMEM (two
//                        256-column accumulators, so the epilogue of a tile overlaps the main loop of
//                        the next); four epilogue warps per CTA read them with tcgen05.ld.
//   gemm_bf16_kernel     the same on one SM per 128 x 256 tile (four-stage ring of 16 + 32 KB, SS
//                        tcgen05.mma M128 N256 K16), for at most 128 rows.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "quant.cuh"

namespace nomas {

// ------------------------------------------------------------------------------------------------
// weight quantiser and dequantiser
// ------------------------------------------------------------------------------------------------

constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads) w8_quantize_kernel(const __nv_bfloat16 *w, int64_t k_in,
                                                                    int64_t ldw, int8_t *codes, float *scales) {
    __shared__ float red[kQuantThreads / 32];
    const int64_t n = blockIdx.x;
    const __nv_bfloat16 *row = w + n * ldw;
    float a = 0.0f;
    for (int64_t k = threadIdx.x; k < k_in; k += kQuantThreads) a = fmaxf(a, fabsf(__bfloat162float(row[k])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    a = red[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) a = fmaxf(a, red[i]);
    const float s = div127(a);
    if (threadIdx.x == 0) scales[n] = s;
    const float r = s >= 0x1p-125f ? recip_nr(s) : __int_as_float(0x7fffffff);
    int8_t *out = codes + n * k_in;
    for (int64_t k = threadIdx.x; k < k_in; k += kQuantThreads)
        out[k] = s > 0.0f ? (int8_t)code_of(__bfloat162float(row[k]), s, r) : (int8_t)0;
}

__global__ void __launch_bounds__(256) w8_dequant_kernel(const int8_t *codes, const float *scales, int64_t k_in,
                                                         int64_t total16, __nv_bfloat16 *w) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total16; i += stride) {
        const int64_t e0 = i * 16;                      // K is a multiple of 16 here: one row per group
        const float s = __ldg(scales + e0 / k_in);
        const uint4 c = __ldg(reinterpret_cast<const uint4 *>(codes + e0));
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t word = cw[j >> 1] >> (16 * (j & 1));
            const float lo = __fmul_rn((float)(int8_t)(word & 0xFF), s);
            const float hi = __fmul_rn((float)(int8_t)((word >> 8) & 0xFF), s);
            const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
            o[j] = *reinterpret_cast<const uint32_t *>(&b);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(w + e0);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// Rows whose K is not a multiple of 16: one weight per thread.
__global__ void w8_dequant_tail_kernel(const int8_t *codes, const float *scales, int64_t k_in, int64_t total,
                                       __nv_bfloat16 *w) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride)
        w[i] = __float2bfloat16_rn(__fmul_rn((float)codes[i], __ldg(scales + i / k_in)));
}

// ------------------------------------------------------------------------------------------------
// bf16 GEMM on the tensor cores
// ------------------------------------------------------------------------------------------------

constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 64, kGemmStages = 4;
constexpr int kGemmThreads = 192;           // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue

struct GemmCfg {
    static constexpr int A_STAGE = kGemmBM * kGemmBK * 2;          // 16 KB
    static constexpr int B_STAGE = kGemmBN * kGemmBK * 2;          // 32 KB
    static constexpr int STAGE = A_STAGE + B_STAGE;
    static constexpr int OFF_BAR = kGemmStages * STAGE;
    // full, empty [kGemmStages]; acc_full, acc_empty [2]; mma_done
    static constexpr int NBAR = 2 * kGemmStages + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 32;
    static constexpr int SMEM = BYTES + 1024;                      // slack for 1024-byte alignment
};

struct GemmParams {
    int64_t M, N;
    int32_t k_iters;                        // ceil(K / 64)
    int32_t n_nblk;                         // ceil(N / 256)
    int64_t n_tiles;
    void *y;
    int64_t ldy;
    int32_t y_bf16;
    int32_t y_vec;                          // 16-byte row stores possible (pitch and base aligned)
    int *err;
    uint64_t timeout_ns;
};

// Columns [col, col + 32) of output row `row` from 32 fp32 accumulator values (bf16 or fp32, 16-byte
// stores when the whole run is inside N and the pitch allows).
__device__ __forceinline__ void store_row32(const GemmParams &p, const uint32_t (&r)[32], int64_t row, int64_t col) {
    const bool whole = p.y_vec && col + 32 <= p.N;
    if (p.y_bf16) {
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.y) + row * p.ldy + col;
        if (whole) {
            uint32_t o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                o[i] = *reinterpret_cast<const uint32_t *>(&b);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                reinterpret_cast<uint4 *>(dst)[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        } else {
            for (int i = 0; i < 32 && col + i < p.N; ++i) dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
        }
    } else {
        float *dst = static_cast<float *>(p.y) + row * p.ldy + col;
        if (whole) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                reinterpret_cast<float4 *>(dst)[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                                 __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        } else {
            for (int i = 0; i < 32 && col + i < p.N; ++i) dst[i] = __uint_as_float(r[i]);
        }
    }
}

// Tile t of the persistent schedule: N blocks fastest, so the CTAs running at one time share a few
// A row blocks and sweep B (which the 126 MB L2 holds for the DiT's shapes).
__device__ __forceinline__ void gemm_tile(const GemmParams &p, int64_t t, int &mb, int &nb) {
    mb = (int)(t / p.n_nblk);
    nb = (int)(t - (int64_t)mb * p.n_nblk);
}

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_bf16_kernel(const __grid_constant__ CUtensorMap ta,
                                                                     const __grid_constant__ CUtensorMap tb,
                                                                     const GemmParams p) {
    using C = GemmCfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *full = bars, *empty = bars + kGemmStages;
    uint64_t *acc_full = empty + kGemmStages, *acc_empty = acc_full + 2, *mma_done = acc_empty + 2;
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kGemmStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);   // the epilogue warps
        }
        mbar_init(mma_done, 1);
        misc[1] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc[0], 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    Watchdog wd{p.err, abort_flag, p.timeout_ns, 9};

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer
            prefetch_tmap(&ta);
            prefetch_tmap(&tb);
            uint32_t issued = 0, par = 0;
            int s = 0, ph = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x) {
                int mb, nb;
                gemm_tile(p, t, mb, nb);
                for (int kb = 0; kb < p.k_iters; ++kb) {
                    if (!(ok = mbar_wait(&empty[s], ph ^ 1, wd, 1))) break;
                    uint8_t *a = sm + s * C::STAGE;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_3d(a, &ta, &full[s], kb * kGemmBK, mb * kGemmBM, 0);
                    tma_load_3d(a + C::A_STAGE, &tb, &full[s], kb * kGemmBK, nb * kGemmBN, 0);
                    issued |= 1u << s;
                    par = (par & ~(1u << s)) | ((uint32_t)ph << s);
                    if (++s == kGemmStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // copies in flight must land before the CTA's shared memory is released (abort path)
            for (int i = 0; i < kGemmStages; ++i)
                if ((issued >> i) & 1u) mbar_drain(&full[i], (par >> i) & 1u, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, kGemmBN);
            const uint64_t d0 = sdesc_sw128(smem_u32(sm), 16, 1024);   // + byte offset / 16 per stage, K step
            int s = 0, ph = 0, acc = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x, ++acc) {
                const int buf = acc & 1;
                if (!(ok = mbar_wait(&acc_empty[buf], ((acc >> 1) & 1) ^ 1, wd, 2))) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * kGemmBN);
                for (int kb = 0; kb < p.k_iters; ++kb) {
                    if (!(ok = mbar_wait(&full[s], ph, wd, 3))) break;
                    tc_fence_after();
                    const uint64_t da = d0 + (uint64_t)((s * C::STAGE) >> 4);
                    const uint64_t db = da + (uint64_t)(C::A_STAGE >> 4);
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_ss(d, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);      // the stage is free once these MMAs have read it
                    if (++s == kGemmStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit(&acc_full[buf]);
            }
            // every MMA must be complete before TMEM is released, also on the abort path
            umma_commit(mma_done);
            mbar_drain(mma_done, 0, 100000000ull);
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------------- epilogue warps 2-5
        const int g = warp & 3;                          // TMEM lane group (warps 2, 3, 4, 5 -> 2, 3, 0, 1)
        const uint32_t lane_base = (uint32_t)(g * 32) << 16;
        int acc = 0;
        for (int64_t t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++acc) {
            const int buf = acc & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (acc >> 1) & 1, wd, 4))) break;
            tc_fence_after();
            int mb, nb;
            gemm_tile(p, t, mb, nb);
            const int64_t row = (int64_t)mb * kGemmBM + g * 32 + lane;
            const bool row_ok = row < p.M;
            const int64_t col0 = (int64_t)nb * kGemmBN;
#pragma unroll 1
            for (int c0 = 0; c0 < kGemmBN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32_sync(tmem + lane_base + (uint32_t)(buf * kGemmBN + c0), r);
                const int64_t col = col0 + c0;
                if (!row_ok || col >= p.N) continue;
                store_row32(p, r, row, col);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);   // this warp's rows of the accumulator are read
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------------
// bf16 GEMM on SM pairs (cta_group::2)
// ------------------------------------------------------------------------------------------------
// A cluster of two CTAs on an SM pair computes a 256 x 256 tile: each CTA stages 128 rows of A and 128
// rows (output columns) of B per K step, and one tcgen05.mma.cta_group::2 of M256 N256 K16, issued by
// the even CTA, reads both CTAs' halves and accumulates rows 0..127 in the even CTA's TMEM and rows
// 128..255 in the odd one's.  Per SM this moves 32 KB of operands per K step of 64 instead of the
// 48 KB of the one-SM 128 x 256 tile for the same MMA work.
//   full[s]      even CTA only: one arrive_expect_tx of both CTAs' bytes; both CTAs' copies complete on it
//   empty[s]     each CTA: the even CTA's MMA commit, multicast to both, frees the stage
//   acc_full[b]  each CTA: the MMA commit of a tile, multicast to both
//   acc_empty[b] even CTA only: the four epilogue warps of both CTAs arrive (eight)
constexpr int kG2Stages = 6;
constexpr uint16_t kPairMask = 0x3;

struct Gemm2Cfg {
    static constexpr int A_STAGE = 128 * kGemmBK * 2;              // 16 KB: this CTA's 128 rows of A
    static constexpr int B_STAGE = 128 * kGemmBK * 2;              // 16 KB: this CTA's 128 rows of B
    static constexpr int STAGE = A_STAGE + B_STAGE;
    static constexpr int OFF_BAR = kG2Stages * STAGE;
    // full, empty [kG2Stages]; acc_full, acc_empty [2]; mma_done
    static constexpr int NBAR = 2 * kG2Stages + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 32;
    static constexpr int SMEM = BYTES + 1024;
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the even CTA's copy of a barrier of this CTA (same offset): its shared::cluster address
__device__ __forceinline__ uint32_t even_cta_addr(const void *p) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(smem_u32(p)));
    return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// a TMA box into this CTA's shared memory whose bytes complete on the even CTA's barrier
__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on the barrier at this offset in both CTAs once the MMAs issued so far have completed
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(kPairMask)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Tile t of a pair's persistent schedule: 256 x 256, N blocks fastest.
__device__ __forceinline__ void gemm2_tile(const GemmParams &p, int64_t t, int &mb, int &nb) {
    mb = (int)(t / p.n_nblk);
    nb = (int)(t - (int64_t)mb * p.n_nblk);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm2_bf16_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                      const GemmParams p) {
    using C = Gemm2Cfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *full = bars, *empty = bars + kG2Stages;
    uint64_t *acc_full = empty + kG2Stages, *acc_empty = acc_full + 2, *mma_done = acc_empty + 2;
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool even = rank == 0;
    const int64_t pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kG2Stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);   // the epilogue warps of both CTAs
        }
        mbar_init(mma_done, 1);
        misc[1] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&misc[0], 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();                    // both CTAs' barriers are initialised before any remote use
    tc_fence_after();
    const uint32_t tmem = misc[0];
    Watchdog wd{p.err, abort_flag, p.timeout_ns, 9};

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer (both CTAs)
            prefetch_tmap(&ta);
            prefetch_tmap(&tb);
            uint32_t issued = 0, par = 0;
            int s = 0, ph = 0;
            bool ok = true;
            for (int64_t t = pair; ok && t < p.n_tiles; t += n_pairs) {
                int mb, nb;
                gemm2_tile(p, t, mb, nb);
                for (int kb = 0; kb < p.k_iters; ++kb) {
                    if (!(ok = mbar_wait(&empty[s], ph ^ 1, wd, 1))) break;
                    uint8_t *a = sm + s * C::STAGE;
                    if (even) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE);
                    const uint32_t fb = even_cta_addr(&full[s]);
                    tma_load_3d_pair(a, &ta, fb, kb * kGemmBK, mb * 256 + (int)rank * 128, 0);
                    tma_load_3d_pair(a + C::A_STAGE, &tb, fb, kb * kGemmBK, nb * 256 + (int)rank * 128, 0);
                    issued |= 1u << s;
                    par = (par & ~(1u << s)) | ((uint32_t)ph << s);
                    if (++s == kG2Stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // the even CTA's full barriers count both CTAs' bytes: it drains them before the final
            // cluster barrier, which the odd CTA passes only after (abort path)
            if (even)
                for (int i = 0; i < kG2Stages; ++i)
                    if ((issued >> i) & 1u) mbar_drain(&full[i], (par >> i) & 1u, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (even && lane == 0) {
            // ------------------------------------------------------------ MMA issuer (even CTA)
            constexpr uint32_t idesc = idesc_bf16_f32(256, kGemmBN);
            const uint64_t d0 = sdesc_sw128(smem_u32(sm), 16, 1024);
            int s = 0, ph = 0, acc = 0;
            bool ok = true;
            for (int64_t t = pair; ok && t < p.n_tiles; t += n_pairs, ++acc) {
                const int buf = acc & 1;
                if (!(ok = mbar_wait(&acc_empty[buf], ((acc >> 1) & 1) ^ 1, wd, 2))) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * kGemmBN);
                for (int kb = 0; kb < p.k_iters; ++kb) {
                    if (!(ok = mbar_wait(&full[s], ph, wd, 3))) break;
                    tc_fence_after();
                    const uint64_t da = d0 + (uint64_t)((s * C::STAGE) >> 4);
                    const uint64_t db = da + (uint64_t)(C::A_STAGE >> 4);
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_ss_pair(d, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc,
                                     (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair(&empty[s]);
                    if (++s == kG2Stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit_pair(&acc_full[buf]);
            }
            // every MMA must be complete before either CTA releases TMEM or shared memory
            umma_commit_pair(mma_done);
            mbar_drain(mma_done, 0, 100000000ull);
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------------- epilogue warps 2-5 (both CTAs)
        const int g = warp & 3;
        const uint32_t lane_base = (uint32_t)(g * 32) << 16;
        int acc = 0;
        for (int64_t t = pair; t < p.n_tiles; t += n_pairs, ++acc) {
            const int buf = acc & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (acc >> 1) & 1, wd, 4))) break;
            tc_fence_after();
            int mb, nb;
            gemm2_tile(p, t, mb, nb);
            const int64_t row = (int64_t)mb * 256 + (int64_t)rank * 128 + g * 32 + lane;
            const bool row_ok = row < p.M;
            const int64_t col0 = (int64_t)nb * kGemmBN;
#pragma unroll 1
            for (int c0 = 0; c0 < kGemmBN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32_sync(tmem + lane_base + (uint32_t)(buf * kGemmBN + c0), r);
                const int64_t col = col0 + c0;
                if (!row_ok || col >= p.N) continue;
                store_row32(p, r, row, col);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(even_cta_addr(&acc_empty[buf]));
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                    // the even CTA's MMAs are done with both CTAs' memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

}  // namespace nomas

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
namespace nomas {

static bool pitch_ok(int64_t ld, int64_t k) { return ld >= k && ld % 8 == 0; }

static int gemm_attr() {
    static std::once_flag once;
    static cudaError_t e = cudaSuccess;
    std::call_once(once, [] {
        e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemm2_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Gemm2Cfg::SMEM);
    });
    return e == cudaSuccess ? NOMAS_OK : cuda_fail("cudaFuncSetAttribute(gemm smem)", (int)e, cudaGetErrorString(e));
}

static int check_linear(const void *x, int64_t m, int64_t k_in, int64_t ldx, const void *w, int64_t n_out,
                        void *y, int64_t ldy, int y_dtype, int32_t *status) {
    if (!x || !w || !y || !status || !aligned16(x) || !aligned16(w) || !aligned16(y) || !aligned16(status))
        return NOMAS_EINVAL;
    if (m < 1 || n_out < 1 || k_in < 8 || k_in % 8 != 0 || !pitch_ok(ldx, k_in) || ldy < n_out)
        return NOMAS_EINVAL;
    if (y_dtype != NOMAS_DTYPE_F32 && y_dtype != NOMAS_DTYPE_BF16) return NOMAS_EINVAL;
    if (m > ((int64_t)1 << 31) || n_out > ((int64_t)1 << 31)) return NOMAS_EUNSUPPORTED;
    return NOMAS_OK;
}

static int enqueue_linear(const void *x, int64_t m, int64_t k_in, int64_t ldx, const void *w, int64_t n_out,
                          int64_t ldw, void *y, int64_t ldy, int y_dtype, int32_t *status, cudaStream_t st) {
    if (gemm_attr()) return NOMAS_ECUDA;
    CUtensorMap ta, tb;
    const cuuint64_t da[3] = {(cuuint64_t)k_in, (cuuint64_t)m, 1};
    const cuuint64_t sa[2] = {(cuuint64_t)ldx * 2, (cuuint64_t)ldx * 2 * (cuuint64_t)m};
    // SM pairs (256 x 256 tiles, 128 rows of A and of B per CTA) unless there is one pair's worth of rows
    // or less; then one SM per 128 x 256 tile
    const bool pair = m > 128 && sm_count() >= 2;
    const cuuint32_t ba[3] = {kGemmBK, kGemmBM, 1};
    const cuuint64_t db[3] = {(cuuint64_t)k_in, (cuuint64_t)n_out, 1};
    const cuuint64_t sb[2] = {(cuuint64_t)ldw * 2, (cuuint64_t)ldw * 2 * (cuuint64_t)n_out};
    const cuuint32_t bb[3] = {kGemmBK, pair ? 128u : (cuuint32_t)kGemmBN, 1};
    if (!make_tensor_map_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, da, sa, ba, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tensor_map_3d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_128B))
        return NOMAS_ECUDA;
    GemmParams p{};
    p.M = m;
    p.N = n_out;
    p.k_iters = (int32_t)((k_in + kGemmBK - 1) / kGemmBK);
    p.n_nblk = (int32_t)((n_out + kGemmBN - 1) / kGemmBN);
    p.n_tiles = (int64_t)p.n_nblk * ((m + (pair ? 256 : kGemmBM) - 1) / (pair ? 256 : kGemmBM));
    p.y = y;
    p.ldy = ldy;
    p.y_bf16 = y_dtype == NOMAS_DTYPE_BF16;
    p.y_vec = ldy % (p.y_bf16 ? 8 : 4) == 0;
    p.err = status;
    p.timeout_ns = wait_limit_ns();
    if (pair) {
        int64_t pairs = sm_count() / 2;
        if (pairs > p.n_tiles) pairs = p.n_tiles;
        gemm2_bf16_kernel<<<(unsigned)(2 * pairs), kGemmThreads, Gemm2Cfg::SMEM, st>>>(ta, tb, p);
        return check_launch("gemm2_bf16_kernel launch");
    }
    int64_t grid = sm_count();
    if (grid > p.n_tiles) grid = p.n_tiles;
    gemm_bf16_kernel<<<(unsigned)grid, kGemmThreads, GemmCfg::SMEM, st>>>(ta, tb, p);
    return check_launch("gemm_bf16_kernel launch");
}

static int enqueue_dequant(const int8_t *codes, const float *scales, int64_t n_out, int64_t k_in, void *w,
                           cudaStream_t st) {
    const int64_t total = n_out * k_in;
    auto *out = static_cast<__nv_bfloat16 *>(w);
    if (k_in % 16 == 0) {
        const int64_t groups = total / 16;
        int64_t blocks = (groups + 255) / 256;
        if (blocks > (int64_t)sm_count() * 8) blocks = (int64_t)sm_count() * 8;
        w8_dequant_kernel<<<(unsigned)blocks, 256, 0, st>>>(codes, scales, k_in, groups, out);
    } else {
        int64_t blocks = (total + 255) / 256;
        if (blocks > (int64_t)sm_count() * 8) blocks = (int64_t)sm_count() * 8;
        w8_dequant_tail_kernel<<<(unsigned)blocks, 256, 0, st>>>(codes, scales, k_in, total, out);
    }
    return check_launch("w8_dequant_kernel launch");
}

}  // namespace nomas

using namespace nomas;

extern "C" int nomas_w8_quantize(const void *w, int64_t n_out, int64_t k_in, int64_t ldw, int8_t *codes,
                                 float *scales, nomas_stream stream) {
    if (!w || !codes || !scales || n_out < 1 || k_in < 1 || ldw < k_in) return NOMAS_EINVAL;
    if (n_out > ((int64_t)1 << 31) - 1) return NOMAS_EUNSUPPORTED;
    w8_quantize_kernel<<<(unsigned)n_out, kQuantThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(w), k_in, ldw, codes, scales);
    return check_launch("w8_quantize_kernel launch");
}

extern "C" int nomas_w8_dequant(const int8_t *codes, const float *scales, int64_t n_out, int64_t k_in, void *w,
                                nomas_stream stream) {
    if (!codes || !scales || !w || !aligned16(codes) || !aligned16(w) || n_out < 1 || k_in < 8 || k_in % 8 != 0)
        return NOMAS_EINVAL;
    return enqueue_dequant(codes, scales, n_out, k_in, w, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int nomas_linear_bf16(const void *x, int64_t m, int64_t k_in, int64_t ldx, const void *w, int64_t n_out,
                                 int64_t ldw, void *y, int64_t ldy, int y_dtype, int32_t *status, nomas_stream stream) {
    int rc = check_linear(x, m, k_in, ldx, w, n_out, y, ldy, y_dtype, status);
    if (rc) return rc;
    if (!pitch_ok(ldw, k_in)) return NOMAS_EINVAL;
    return enqueue_linear(x, m, k_in, ldx, w, n_out, ldw, y, ldy, y_dtype, reinterpret_cast<int *>(status),
                          reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t nomas_w8a16_workspace_bytes(int64_t n_out, int64_t k_in) {
    if (n_out < 1 || k_in < 1) return 0;
    return (size_t)n_out * (size_t)k_in * 2;
}

extern "C" int nomas_w8a16_linear(const void *x, int64_t m, int64_t k_in, int64_t ldx, const int8_t *codes,
                                  const float *scales, int64_t n_out, void *y, int64_t ldy, int y_dtype,
                                  void *workspace, int32_t *status, nomas_stream stream) {
    int rc = check_linear(x, m, k_in, ldx, workspace, n_out, y, ldy, y_dtype, status);
    if (rc) return rc;
    if (!codes || !scales || !aligned16(codes)) return NOMAS_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (gemm_attr()) return NOMAS_ECUDA;
    rc = enqueue_dequant(codes, scales, n_out, k_in, workspace, st);
    if (rc) return rc;
    return enqueue_linear(x, m, k_in, ldx, workspace, n_out, k_in, y, ldy, y_dtype, reinterpret_cast<int *>(status), st);
}

extern "C" int nomas_status_read(int32_t *status, nomas_stream stream) {
    if (!status) return NOMAS_EINVAL;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NOMAS_ECUDA;
    int32_t w[4] = {0, 0, 0, 0};
    if (cudaMemcpy(w, status, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return NOMAS_ECUDA;
    if (w[0] != 0) {
        if (cudaMemset(status, 0, sizeof(w)) != cudaSuccess) return NOMAS_ECUDA;
        return w[0];
    }
    return NOMAS_OK;
}
