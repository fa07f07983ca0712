// Archive of evicted history frames and selection of the retained history (hyphentech.top config
// table: the GPU keeps at most 18 history latent frames, earlier history is archived to CPU).  The
// reading, the record layout and the limits are stated in nomas.h.  Only host code: the copies between
// the ring and host records are strided 2-D memory copies (one per buffer and frame, the heads as rows).
#include <vector>

#include "common.cuh"

namespace nomas {

struct RecordLayout {
    size_t k8, v8, ks, vs, total;   // byte offsets inside one record
};

static RecordLayout record_layout(const nomas_cache_dims &d) {
    const size_t codes = (size_t)d.heads * d.tokens_per_frame * d.head_dim;
    const size_t scales = (size_t)d.heads * d.tokens_per_frame * sizeof(float);
    return RecordLayout{0, codes, 2 * codes, 2 * codes + scales, 2 * codes + 2 * scales};
}

// Copy frame slot `slot` of the ring to (to_host) or from a record: per buffer one 2-D copy whose rows
// are the heads (ring rows of a head are C * T apart, a record's are T apart).
static int copy_frame(const nomas_kv_cache *c, int32_t slot, void *record, bool to_host, cudaStream_t st) {
    const auto &d = c->d;
    const RecordLayout L = record_layout(d);
    const size_t T = d.tokens_per_frame, D = d.head_dim, C = d.capacity_frames;
    uint8_t *rec = static_cast<uint8_t *>(record);
    struct Part {
        int buf;
        size_t off, elem, row_elems;   // record offset, element bytes, elements of one head's frame
    };
    const Part parts[4] = {{NOMAS_BUF_K8, L.k8, 1, T * D}, {NOMAS_BUF_V8, L.v8, 1, T * D},
                           {NOMAS_BUF_KS, L.ks, 4, T}, {NOMAS_BUF_VS, L.vs, 4, T}};
    for (const Part &pt : parts) {
        uint8_t *ring = static_cast<uint8_t *>(c->buf[pt.buf]) + (size_t)slot * pt.row_elems * pt.elem;
        const size_t width = pt.row_elems * pt.elem, ring_pitch = C * pt.row_elems * pt.elem;
        const cudaError_t e =
            to_host ? cudaMemcpy2DAsync(rec + pt.off, width, ring, ring_pitch, width, (size_t)d.heads,
                                        cudaMemcpyDeviceToHost, st)
                    : cudaMemcpy2DAsync(ring, ring_pitch, rec + pt.off, width, width, (size_t)d.heads,
                                        cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return cuda_fail("cudaMemcpy2DAsync(frame record)", (int)e, cudaGetErrorString(e));
    }
    return NOMAS_OK;
}

static int retained_index(const nomas_kv_cache *c, int64_t frame) {
    for (size_t i = 0; i < c->ret_frame.size(); ++i)
        if (c->ret_frame[i] == frame) return (int)i;
    return -1;
}

}  // namespace nomas

using namespace nomas;

extern "C" size_t nomas_kv_frame_record_bytes(const nomas_cache_dims *dims) {
    if (nomas_kv_cache_bytes(dims, nullptr) == 0) return 0;
    return record_layout(*dims).total;
}

extern "C" int nomas_kv_retained(const nomas_kv_cache *c, int64_t *frames, int32_t max_frames, int32_t *n) {
    if (!c || !n || max_frames < 0 || (max_frames > 0 && !frames)) return NOMAS_EINVAL;
    const int32_t cnt = (int32_t)c->ret_frame.size();
    *n = cnt;
    if (cnt > max_frames) return NOMAS_ECAPACITY;
    for (int32_t i = 0; i < cnt; ++i) frames[i] = c->ret_frame[i];
    return NOMAS_OK;
}

extern "C" int nomas_kv_evicted_by(const nomas_kv_cache *c, int32_t n_frames, int64_t *frames, int32_t max_frames,
                                   int32_t *n) {
    if (!c || !n || n_frames < 0 || max_frames < 0 || (max_frames > 0 && !frames)) return NOMAS_EINVAL;
    const auto &d = c->d;
    int64_t drop = 0;
    if (d.window_frames > 0) {
        const int64_t keep = n_frames < d.window_frames ? n_frames : d.window_frames;
        drop = (int64_t)c->ret_frame.size() + keep - d.window_frames;
        if (drop < 0) drop = 0;
    }
    *n = (int32_t)drop;
    if (drop > max_frames) return NOMAS_ECAPACITY;
    for (int64_t i = 0; i < drop; ++i) frames[i] = c->ret_frame[(size_t)i];
    return NOMAS_OK;
}

extern "C" int nomas_kv_archive(const nomas_kv_cache *c, int64_t frame, void *record, nomas_stream stream) {
    if (!c || !record) return NOMAS_EINVAL;
    const int i = retained_index(c, frame);
    if (i < 0) return NOMAS_EINVAL;
    if (bind_device(c)) return NOMAS_ECUDA;
    return copy_frame(c, c->ret_slot[(size_t)i], record, true, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int nomas_kv_select(nomas_kv_cache *c, const int64_t *frames, int32_t n, const void *const *records,
                               nomas_stream stream) {
    if (!c || n < 0 || (n > 0 && !frames)) return NOMAS_EINVAL;
    const auto &d = c->d;
    if (d.window_frames == 0 || d.window_frames > NOMAS_MAX_SELECT_FRAMES) return NOMAS_EUNSUPPORTED;
    if (n > d.window_frames) return NOMAS_EINVAL;
    // validate everything before the first copy: no repeat, a record for every frame not retained
    std::vector<int> where((size_t)n);
    for (int32_t i = 0; i < n; ++i) {
        for (int32_t j = 0; j < i; ++j)
            if (frames[j] == frames[i]) return NOMAS_EINVAL;
        where[(size_t)i] = retained_index(c, frames[i]);
        if (where[(size_t)i] < 0 && (!records || !records[i])) return NOMAS_EINVAL;
    }
    // slots: kept frames keep theirs; incoming frames take free slots, first those no retained frame
    // holds (so the current history survives as long as possible), then those of dropped frames
    const int32_t C = d.capacity_frames;
    std::vector<char> kept_slot((size_t)C, 0), cur_slot((size_t)C, 0);
    for (int32_t sl : c->ret_slot) cur_slot[(size_t)sl] = 1;
    for (int32_t i = 0; i < n; ++i)
        if (where[(size_t)i] >= 0) kept_slot[(size_t)c->ret_slot[(size_t)where[(size_t)i]]] = 1;
    std::vector<int32_t> slot((size_t)n);
    std::vector<char> taken(kept_slot);
    for (int32_t i = 0; i < n; ++i) {
        if (where[(size_t)i] >= 0) {
            slot[(size_t)i] = c->ret_slot[(size_t)where[(size_t)i]];
            continue;
        }
        int32_t s = -1;
        for (int32_t k = 0; k < C && s < 0; ++k)
            if (!taken[(size_t)k] && !cur_slot[(size_t)k]) s = k;
        for (int32_t k = 0; k < C && s < 0; ++k)
            if (!taken[(size_t)k]) s = k;
        taken[(size_t)s] = 1;   // exists: n <= W <= C
        slot[(size_t)i] = s;
    }
    if (bind_device(c)) return NOMAS_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int32_t i = 0; i < n; ++i) {
        if (where[(size_t)i] >= 0) continue;
        const int rc = copy_frame(c, slot[(size_t)i], const_cast<void *>(records[i]), false, st);
        if (rc) return rc;
    }
    c->ret_frame.assign(frames, frames + n);
    c->ret_slot = slot;
    c->version += 1;
    return NOMAS_OK;
}
