// Pre-pass of nomas_attn_fwd (HBM-bound): operand copies in the layouts the attention kernel's TMA
// boxes read -- fp16 keys [H][n][D], fp16 values transposed [H][D][n], and the cache's INT8 codes
// widened to exact fp16 in the same layouts.
#pragma once

#include "common.cuh"

namespace nomas {

// bf16 [n][H][D] (token / head strides in elements) -> fp16 [H][n][D], for up to two tensors.
struct F16Job {
    const __nv_bfloat16 *src;
    __half *dst;
    int64_t n;
};
struct F16Jobs {
    F16Job job[2];
    int32_t n_jobs;
    int32_t H, D;
    int64_t tok_stride, head_stride;
    int *err;            // device error word: NOMAS_ERANGE for a value outside the fp16 range
    WsHeader hdr;        // written to *hdr_dst by the first block
    WsHeader *hdr_dst;
};

// bf16 [n][H][D] -> fp16 V^T [H][D][np] (np = n rounded up to 8, zero padding); job[1] is used when
// `two` is set.
struct VtJob {
    const __nv_bfloat16 *src;
    __half *dst;
    int64_t n, np;
};
struct VtJobs {
    VtJob job[2];
    int32_t H, D;
    int64_t tok_stride, head_stride;
    int *err;            // device error word: NOMAS_ERANGE for a value outside the fp16 range
};

// INT8 ring rows of the retained history (age order) and description-head rows -> fp16 codes; see
// the history part of prepare_kernel.
struct HistPrep {
    const int8_t *k8, *v8, *hk8, *hv8;
    const float *ks, *vs;
    __half *kh, *vht, *kp, *vpt;
    float *ksl, *vsl;
    const float *hks, *hvs;   // description-head scales (checked only)
    HistView hv;              // ring rows of the retained history in age order
    int64_t Lh, lhp, Lp, lpp, head_rows;
    int32_t H, D;
    int *err;                 // device error word: NOMAS_ERANGE for a value scale above kMaxValueScale
};

// One launch for the three copies of a call (keys, transposed values, and -- when hp is not null -- the
// retained history and the description heads); returns NOMAS_OK or the launch error.
int launch_prepare(const F16Jobs &fj, const VtJobs &vj, bool two, int64_t max_np, const HistPrep *hp, cudaStream_t st);

}  // namespace nomas
