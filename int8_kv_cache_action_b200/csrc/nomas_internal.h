// Internal declarations shared by the libnomas translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <vector>

#include "nomas.h"

struct nomas_kv_cache {
    nomas_cache_dims d;
    void *buf[NOMAS_NBUF];
    int64_t frames_appended;
    int64_t head_used;
    int64_t version;                   // changes with every append and selection (checked by the kernels)
    int32_t segments;
    int32_t device;                    // CUDA device owning the buffers; made current on every call
    std::vector<int64_t> ret_frame;    // retained history frames (global index), age order
    std::vector<int32_t> ret_slot;     // their ring slots
};

namespace nomas {

constexpr int kTile = 128;                 // query block and KV tile size
constexpr uint32_t kMaskMagic = 0x4E4D534Bu;
constexpr int32_t kAlwaysHi = 1 << 30;      // 'visible to every frame' upper window bound

// Ring view of the retained history in age order (host-computed, passed by value to kernels).  Without
// a selection the retained frames sit in consecutive slots (frame g in slot g mod C); after
// nomas_kv_select they may sit anywhere, and the slot of every frame is listed.
struct HistView {
    int64_t ring_tokens;     // C * T
    int64_t first_tok;       // contiguous: physical token of the oldest retained token
    int64_t tokens;          // retained history tokens
    int32_t T;
    int32_t contiguous;      // 1: frame i of the history is in slot (first slot + i) mod C
    int32_t n_frames;
    int32_t slots[NOMAS_MAX_SELECT_FRAMES];   // otherwise: slot of history frame i (n_frames <= the max)
};

inline HistView hist_view(const nomas_kv_cache *c) {
    const auto &d = c->d;
    HistView v{};
    const int n = (int)c->ret_slot.size();
    v.ring_tokens = (int64_t)d.capacity_frames * d.tokens_per_frame;
    v.tokens = (int64_t)n * d.tokens_per_frame;
    v.T = d.tokens_per_frame;
    v.n_frames = n;
    v.contiguous = 1;
    for (int i = 1; i < n; ++i)
        if (c->ret_slot[i] != (c->ret_slot[0] + i) % d.capacity_frames) v.contiguous = 0;
    v.first_tok = n ? (int64_t)c->ret_slot[0] * d.tokens_per_frame : 0;
    if (!v.contiguous)
        for (int i = 0; i < n && i < NOMAS_MAX_SELECT_FRAMES; ++i) v.slots[i] = c->ret_slot[i];
    return v;
}

// Physical ring row (within one head) of history token a (age order).
#if defined(__CUDACC__)
__host__ __device__ __forceinline__
#else
inline
#endif
int64_t hist_row(const HistView &v, int64_t a) {
    if (v.contiguous) {
        const int64_t p = v.first_tok + a;   // first_tok < C T and a < C T
        return p >= v.ring_tokens ? p - v.ring_tokens : p;
    }
    const int64_t f = a / v.T;
    return (int64_t)v.slots[f] * v.T + (a - f * v.T);
}

// Division by an invariant divisor d >= 1 for numerators below 2^31 (Granlund and Montgomery,
// "Division by invariant integers using multiplication", 1994): l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (umulhi(n, m) + n) >> l.
struct FastDiv {
    uint32_t d, m, l;
};
inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while (l < 32 && ((uint64_t)1 << l) < d) ++l;
    const uint64_t m = (((uint64_t)1 << 32) * (((uint64_t)1 << l) - d)) / d + 1;
    return FastDiv{d, (uint32_t)m, l};
}

// Visibility codes (fluxbbs.com "架构": action tails visible only in their own segment and time
// window; text query rows: see the reading in nomas.h).  A key and a query row each carry two
// half-open frame intervals, x..y ("video" interval) and z..w ("tail" interval); the key is visible to
// the row iff one of the pairs overlaps:  max(k.x, r.x) < min(k.y, r.y) || max(k.z, r.z) < min(k.w, r.w).
//   key  always visible (history, earlier heads, current head): {-kBig, kBig, kNeg, kBig}
//        current video frame t:                                 {t, t + 1, 0, 0}
//        action tail with window [f0, f1):                      {0, 0, f0, f1}
//        past the end of its tile:                              {0, 0, 0, 0}
//   row  video frame t:                                         {-kBig, kBig, t, t + 1}
//        description-head text row:                             {-kBig, kBig, 0, 0}
//        text row of a tail with window [f0, f1):               {f0, f1, f0, f1}, or {f0, f1, kNeg, kNeg + 1}
//                                                               when the window is empty
constexpr int32_t kBig = 1 << 30;
constexpr int32_t kNeg = -2147483647;   // below every frame and every -kBig

struct VisCode {
    int32_t x, y, z, w;
};

#if defined(__CUDACC__)
#define NOMAS_HD __host__ __device__ __forceinline__
#else
#define NOMAS_HD inline
#endif

NOMAS_HD VisCode key_always() { return VisCode{-kBig, kBig, kNeg, kBig}; }
NOMAS_HD VisCode key_video(int32_t t) { return VisCode{t, t + 1, 0, 0}; }
NOMAS_HD VisCode key_tail(int32_t f0, int32_t f1) { return VisCode{0, 0, f0, f1}; }
NOMAS_HD VisCode key_none() { return VisCode{0, 0, 0, 0}; }
NOMAS_HD VisCode row_video(int32_t t) { return VisCode{-kBig, kBig, t, t + 1}; }
NOMAS_HD VisCode row_head() { return VisCode{-kBig, kBig, 0, 0}; }
NOMAS_HD VisCode row_tail(int32_t f0, int32_t f1) {
    return f0 < f1 ? VisCode{f0, f1, f0, f1} : VisCode{f0, f1, kNeg, kNeg + 1};
}
NOMAS_HD bool visible(const VisCode &k, const VisCode &r) {
    return (k.x > r.x ? k.x : r.x) < (k.y < r.y ? k.y : r.y) || (k.z > r.z ? k.z : r.z) < (k.w < r.w ? k.w : r.w);
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
    int64_t cache_version;
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
    int64_t cache_version;
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
int text_split_setting();   // nomas_set_text_split: 0 = chosen per call, else 1..16
int attn_kernel_setting();  // nomas_set_attn_kernel: 0 = chosen per call, 1 = one block per CTA, 2 = block pairs

}  // namespace nomas
