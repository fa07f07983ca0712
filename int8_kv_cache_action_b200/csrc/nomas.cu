// libnomas host entry points: cache handle, buffer sizes, state, status, mask-buffer layout.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "common.cuh"

namespace nomas {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static thread_local char g_last_error[256] = "";

int cuda_fail(const char *what, int code, const char *detail) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s failed (%d): %s", what, code, detail ? detail : "");
    return NOMAS_ECUDA;
}

int check_launch(const char *what) {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? NOMAS_OK : cuda_fail(what, (int)e, cudaGetErrorString(e));
}

static std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};   // 2 s per wait

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

static std::atomic<int> g_text_split{0};   // 0: chosen per call

int text_split_setting() { return g_text_split.load(std::memory_order_relaxed); }
static std::atomic<int> g_attn_kernel{0};   // 0: chosen per call, 1: one block per CTA, 2: block pairs
int attn_kernel_setting() { return g_attn_kernel.load(std::memory_order_relaxed); }

int bind_device(const nomas_kv_cache *c) {
    int cur = -1;
    if (cudaGetDevice(&cur) == cudaSuccess && cur == c->device) return NOMAS_OK;
    const cudaError_t e = cudaSetDevice(c->device);
    return e == cudaSuccess ? NOMAS_OK : cuda_fail("cudaSetDevice", (int)e, cudaGetErrorString(e));
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load();
    if (!f) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr = cudaDriverEntryPointSymbolNotFound;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr);
        if (e == cudaSuccess && qr == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<EncodeTiledFn>(ptr);
            fn.store(f);
        } else {
            cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", e != cudaSuccess ? (int)e : (int)qr,
                      e != cudaSuccess ? cudaGetErrorString(e) : "symbol query failed");
        }
    }
    return f;
}

bool make_tensor_map_3d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, const cuuint64_t dims[3],
                        const cuuint64_t strides[2], const cuuint32_t box[3], CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint32_t es[3] = {1, 1, 1};
    const CUresult r = enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
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

int sm_count() {
    static std::atomic<int> counts[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = counts[dev].load();
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev].store(n);
    }
    return n;
}

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static bool dims_ok(const nomas_cache_dims *d) {
    if (!d) return false;
    if (d->heads < 1 || d->heads > 1024) return false;
    if (d->head_dim != 64 && d->head_dim != 128) return false;
    if (d->tokens_per_frame < 1 || d->window_frames < 0 || d->capacity_frames < 1 || d->head_store_tokens < 0)
        return false;
    if (d->window_frames > 0 && d->capacity_frames < d->window_frames) return false;
    if ((int64_t)d->capacity_frames * d->tokens_per_frame > (int64_t)1 << 30) return false;
    return true;
}

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int compute_mask_layout(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                        nomas_mask_layout *o) {
    if (!c || !seg || !o) return NOMAS_EINVAL;
    if (mode != NOMAS_MODE_DENSE && mode != NOMAS_MODE_SPARSE && mode != NOMAS_MODE_TEXT) return NOMAS_EINVAL;
    if (seg->n_frames < 1 || seg->head_len < 0 || seg->n_tails < 0 || seg->n_tails > NOMAS_MAX_TAILS)
        return NOMAS_EINVAL;
    if (seg->n_tails > 0 && !seg->tails) return NOMAS_EINVAL;
    int64_t lt = seg->head_len;
    for (int i = 0; i < seg->n_tails; ++i) {
        const nomas_tail &t = seg->tails[i];
        if (t.len < 0 || t.f0 < 0 || t.f1 < t.f0 || t.f1 > seg->n_frames) return NOMAS_EINVAL;
        lt += t.len;
    }
    const auto &d = c->d;
    const HistView hv = hist_view(c);
    std::memset(o, 0, sizeof(*o));
    o->mode = mode;
    o->head_dim = d.head_dim;
    o->heads = d.heads;
    o->history_tokens = hv.tokens;
    o->head_tokens = c->head_used;
    o->n_query = (int64_t)seg->n_frames * d.tokens_per_frame;
    o->text_tokens = lt;
    if (o->n_query > ((int64_t)1 << 30) || lt > ((int64_t)1 << 24)) return NOMAS_EUNSUPPORTED;
    if (mode == NOMAS_MODE_TEXT && lt == 0) return NOMAS_EINVAL;   // no text rows to attend from
    // query blocks: 128 rows of the current video, or of the current text in text mode
    o->n_qblocks = (int32_t)cdiv(mode == NOMAS_MODE_TEXT ? lt : o->n_query, kTile);
    o->n_hist_tiles = (int32_t)cdiv(hv.tokens, kTile);
    o->n_head_tiles = (int32_t)cdiv(c->head_used, kTile);
    o->n_cur_tiles = (int32_t)cdiv(o->n_query, kTile);
    o->n_text_tiles = (int32_t)cdiv(lt, kTile);
    o->n_tiles = o->n_hist_tiles + o->n_head_tiles + o->n_cur_tiles + o->n_text_tiles;
    o->n_cand = o->n_hist_tiles + o->n_cur_tiles;
    if (mode == NOMAS_MODE_SPARSE) {
        if (o->n_cand > NOMAS_MAX_SPARSE_CANDIDATES) return NOMAS_EUNSUPPORTED;
        if (!(keep_frac > 0.0f && keep_frac <= 1.0f)) return NOMAS_EINVAL;
        double k = std::ceil((double)o->n_cand * (double)keep_frac);
        int64_t kk = (int64_t)k;
        if (kk < 1) kk = 1;
        if (kk > o->n_cand) kk = o->n_cand;
        o->keep = (int32_t)kk;
    }
    const int64_t n_pairs = cdiv(o->n_qblocks, 2);
    o->n_lists = (int32_t)(mode == NOMAS_MODE_SPARSE ? n_pairs * d.heads : n_pairs);
    o->list_cap = o->n_tiles;
    const int64_t H = d.heads, D = d.head_dim;
    size_t off = 256;  // MaskHeader
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = round_up(off + bytes, 256);
        return at;
    };
    o->off_class = take((size_t)o->n_qblocks * o->n_tiles);
    const bool sp = mode == NOMAS_MODE_SPARSE;
    o->off_sel = take(sp ? (size_t)H * o->n_qblocks * o->keep * 4 : 0);
    o->off_score = take(sp ? (size_t)H * o->n_qblocks * o->n_cand * 4 : 0);
    o->off_qmean = take(sp ? (size_t)H * o->n_qblocks * D * 4 : 0);
    o->off_kmean = take(sp ? (size_t)H * o->n_cand * D * 4 : 0);
    o->off_txtwin = take((size_t)lt * 8);
    o->off_count = take((size_t)o->n_lists * 4);
    o->off_list = take((size_t)o->n_lists * o->list_cap * 16);
    o->total_bytes = off;
    return NOMAS_OK;
}

}  // namespace nomas

using namespace nomas;

extern "C" size_t nomas_kv_cache_bytes(const nomas_cache_dims *d, size_t out_sizes[NOMAS_NBUF]) {
    if (!dims_ok(d)) return 0;
    const size_t rows = (size_t)d->capacity_frames * d->tokens_per_frame;
    size_t s[NOMAS_NBUF];
    s[NOMAS_BUF_K8] = s[NOMAS_BUF_V8] = round_up((size_t)d->heads * rows * d->head_dim, 16);
    s[NOMAS_BUF_KS] = s[NOMAS_BUF_VS] = round_up((size_t)d->heads * rows * 4, 16);
    s[NOMAS_BUF_HK8] = s[NOMAS_BUF_HV8] = round_up((size_t)d->heads * d->head_store_tokens * d->head_dim, 16);
    s[NOMAS_BUF_HKS] = s[NOMAS_BUF_HVS] = round_up((size_t)d->heads * d->head_store_tokens * 4, 16);
    s[NOMAS_BUF_ERR] = 16;
    size_t tot = 0;
    for (int i = 0; i < NOMAS_NBUF; ++i) {
        tot += s[i];
        if (out_sizes) out_sizes[i] = s[i];
    }
    return tot;
}

extern "C" int nomas_kv_cache_init(nomas_kv_cache **out, const nomas_cache_dims *d, void *const bufs[NOMAS_NBUF],
                                   nomas_stream stream) {
    if (!out || !dims_ok(d) || !bufs) return NOMAS_EINVAL;
    size_t sizes[NOMAS_NBUF];
    nomas_kv_cache_bytes(d, sizes);
    for (int i = 0; i < NOMAS_NBUF; ++i)
        if (sizes[i] > 0 && (!bufs[i] || !aligned16(bufs[i]))) return NOMAS_EINVAL;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, bufs[NOMAS_BUF_ERR]) != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
        cudaGetLastError();
        return NOMAS_EINVAL;
    }
    auto *c = new (std::nothrow) nomas_kv_cache();
    if (!c) return NOMAS_EINVAL;
    c->d = *d;
    for (int i = 0; i < NOMAS_NBUF; ++i) c->buf[i] = bufs[i];
    c->frames_appended = 0;
    c->version = 0;
    c->head_used = 0;
    c->segments = 0;
    c->device = attr.device;
    if (bind_device(c) != NOMAS_OK || cudaMemsetAsync(bufs[NOMAS_BUF_ERR], 0, 16, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        delete c;
        return NOMAS_ECUDA;
    }
    *out = c;
    return NOMAS_OK;
}

extern "C" int nomas_kv_cache_destroy(nomas_kv_cache *c) {
    delete c;
    return NOMAS_OK;
}

extern "C" int nomas_kv_cache_state(const nomas_kv_cache *c, nomas_cache_state *o) {
    if (!c || !o) return NOMAS_EINVAL;
    const HistView hv = hist_view(c);
    std::memset(o, 0, sizeof(*o));
    o->frames_appended = c->frames_appended;
    o->retained_frames = hv.n_frames;
    o->first_slot = hv.n_frames ? c->ret_slot[0] : 0;
    o->history_tokens = hv.tokens;
    o->head_tokens = c->head_used;
    o->segments = c->segments;
    return NOMAS_OK;
}

extern "C" int nomas_mask_layout_query(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode,
                                       float keep_frac, nomas_mask_layout *out) {
    return compute_mask_layout(c, seg, mode, keep_frac, out);
}

extern "C" size_t nomas_mask_bytes(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode,
                                   float keep_frac) {
    nomas_mask_layout l;
    if (compute_mask_layout(c, seg, mode, keep_frac, &l) != NOMAS_OK) return 0;
    return l.total_bytes;
}

extern "C" int nomas_device_status(const nomas_kv_cache *c, nomas_stream stream) {
    if (!c) return NOMAS_EINVAL;
    if (bind_device(c)) return NOMAS_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return NOMAS_ECUDA;
    int w[4] = {0, 0, 0, 0};
    if (cudaMemcpy(w, c->buf[NOMAS_BUF_ERR], sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return NOMAS_ECUDA;
    if (w[0] != 0) {
        if (cudaMemset(c->buf[NOMAS_BUF_ERR], 0, 16) != cudaSuccess) return NOMAS_ECUDA;
        return w[0];
    }
    return NOMAS_OK;
}

extern "C" const char *nomas_last_error(void) { return g_last_error; }

extern "C" uint64_t nomas_set_wait_limit_ns(uint64_t limit_ns) {
    return g_wait_limit_ns.exchange(limit_ns, std::memory_order_relaxed);
}

extern "C" int nomas_set_text_split(int shares) {
    return g_text_split.exchange(shares >= 1 && shares <= 16 ? shares : 0, std::memory_order_relaxed);
}

extern "C" int nomas_set_attn_kernel(int which) {
    return g_attn_kernel.exchange(which == 1 || which == 2 ? which : 0, std::memory_order_relaxed);
}

extern "C" const char *nomas_status_string(int s) {
    switch (s) {
        case NOMAS_OK: return "ok";
        case NOMAS_EINVAL: return "invalid argument";
        case NOMAS_ECAPACITY: return "capacity exceeded";
        case NOMAS_ECUDA: return "CUDA error";
        case NOMAS_ETIMEOUT: return "device wait timed out";
        case NOMAS_EDEVICE: return "inconsistent device data";
        case NOMAS_EUNSUPPORTED: return "unsupported size";
        case NOMAS_ESTATE: return "invalid state";
        case NOMAS_ERANGE: return "attention operand out of range";
        default: return "unknown status";
    }
}
