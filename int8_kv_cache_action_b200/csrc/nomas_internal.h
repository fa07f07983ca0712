// Internal declarations shared by the libnomas translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>

#include "nomas.h"

struct nomas_kv_cache {
    nomas_cache_dims d;
    void *buf[NOMAS_NBUF];
    int64_t frames_appended;
    int64_t head_used;
    int32_t segments;
    int32_t device;          // CUDA device owning the buffers; made current on every call
};

namespace nomas {

constexpr int kTile = 128;                 // query block and KV tile size
constexpr uint32_t kMaskMagic = 0x4E4D534Bu;
constexpr int32_t kAlwaysHi = 1 << 30;      // 'visible to every frame' upper window bound

// Ring view of the retained history (host-computed, passed by value to kernels).
struct HistView {
    int64_t ring_tokens;     // C * T
    int64_t first_tok;       // physical token of the oldest retained token
    int64_t tokens;          // retained history tokens
};

inline HistView hist_view(const nomas_kv_cache *c) {
    const auto &d = c->d;
    int64_t g = c->frames_appended;
    int64_t ret = d.window_frames > 0 ? (g < d.window_frames ? g : d.window_frames) : g;
    int64_t first_frame = g - ret;
    HistView v;
    v.ring_tokens = (int64_t)d.capacity_frames * d.tokens_per_frame;
    v.first_tok = (first_frame % d.capacity_frames) * d.tokens_per_frame;
    v.tokens = ret * d.tokens_per_frame;
    return v;
}

// Per-CTA tile-list entry (int4): x = kind | flags, y = start in its source, z = valid keys, w = spare.
enum TileKind : int { kKindHist = 0, kKindPriorHead = 1, kKindCur = 2, kKindText = 3 };
constexpr int kUse0 = 1 << 2, kUse1 = 1 << 3, kMask0 = 1 << 4, kMask1 = 1 << 5;

// Device header written at offset 0 of the mask buffer; nomas_attn_fwd checks it.
struct MaskHeader {
    uint32_t magic;
    int32_t mode;
    int32_t n_qblocks;
    int32_t n_lists;
    int64_t history_tokens;
    int64_t head_tokens;
    int64_t frames_appended;
    int64_t n_query;
    int64_t text_tokens;
    int32_t list_cap;
    int32_t keep;
};

// Device header written at offset 0 of the attention workspace by nomas_attn_prepare; the attention
// kernel checks it against the cache state and segment of the call.
constexpr uint32_t kWsMagic = 0x4E4D5753u;
struct WsHeader {
    uint32_t magic;
    int32_t head_dim;
    int64_t frames_appended;
    int64_t head_tokens;
    int64_t history_tokens;
    int64_t n_query;
    int64_t text_tokens;
};

int compute_mask_layout(const nomas_kv_cache *c, const nomas_segment_text *seg, int mode, float keep_frac,
                        nomas_mask_layout *out);

bool aligned16(const void *p);

// Record a failing CUDA runtime / driver call for nomas_last_error and return NOMAS_ECUDA.
int cuda_fail(const char *what, int code, const char *detail);
int check_launch(const char *what);

// Make the cache's device current for this thread (the library links its own CUDA runtime).
int bind_device(const nomas_kv_cache *c);

// Limit of every bounded device wait (nomas_set_wait_limit_ns), in nanoseconds.
uint64_t wait_limit_ns();

// Encode a 3-D tiled TMA map (no interleave, L2 256-byte promotion, zero fill out of bounds).  dims /
// box are innermost first, strides in bytes for dims 1 and 2.  Records the failure for
// nomas_last_error and returns false on error.
bool make_tensor_map_3d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, const cuuint64_t dims[3],
                        const cuuint64_t strides[2], const cuuint32_t box[3], CUtensorMapSwizzle swz);

// Number of SMs of the current device (queried once per device).
int sm_count();

}  // namespace nomas
