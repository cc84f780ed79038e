// Shared definitions of the Flint attention kernels: fixed head geometry,
// the workspace layout, the work-item format and the device helpers the
// key-preparation and attention kernels must compute identically.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace flint {

// Head geometry of the Flint attention layer (model page, "Model
// Architecture": 32 query heads, 4 key/value heads, head dimension 128).
constexpr int kHQ = 32;
constexpr int kHKV = 4;
constexpr int kHD = 128;
constexpr int kGroup = kHQ / kHKV;          // query heads per KV head (8)

// Tiling.  One MMA tile of 128 rows packs 16 tokens x the 8 query heads of a
// KV group; a work item is 32 consecutive tokens of one document (two tiles)
// for one KV group; keys are streamed in chunks of 128.
constexpr int kTokPerTile = 16;
constexpr int kTokPerItem = 32;
constexpr int kKeyChunk = 128;

// Device status codes (mirror flint_status_t).
constexpr int kStatusOk = 0;
constexpr int kStatusInvalid = 1;
constexpr int kStatusUnsupported = 2;
constexpr int kStatusTimeout = 4;

enum MaskMode : int { kMaskSingle = 0, kMaskThd = 1, kMaskPad = 2 };

// Workspace layout; all regions 256-byte aligned, the key buffer 1024-byte.
struct WsLayout {
    size_t header, seg, prefix, hist, items, kn, total;
    // FP16 attention-compute policy only (after `total`): the normalised,
    // rotated FP16 queries and the FP16 values
    size_t qn, vh, total_f16;
    int max_items, hist_len;
};

__host__ __device__ inline size_t ws_align(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline WsLayout ws_layout(int T, int nseg) {
    if (nseg < 1) nseg = 1;
    WsLayout L;
    L.max_items = (T + kTokPerItem - 1) / kTokPerItem + nseg + 1;
    L.hist_len = T / kKeyChunk + 3;
    size_t o = 0;
    L.header = o; o += 256;
    L.seg = o;    o = ws_align(o + sizeof(int) * 2 * (size_t)(nseg + 1), 256);
    L.prefix = o; o = ws_align(o + sizeof(int) * (size_t)(nseg + 2), 256);
    L.hist = o;   o = ws_align(o + sizeof(int) * (size_t)L.hist_len, 256);
    L.items = o;  o = ws_align(o + sizeof(int) * 4 * (size_t)L.max_items, 1024);
    L.kn = o;     o = ws_align(o + (size_t)T * kHKV * kHD * 2, 1024);
    L.total = o;
    L.qn = o;     o = ws_align(o + (size_t)T * kHQ * kHD * 2, 1024);
    L.vh = o;     o = ws_align(o + (size_t)T * kHKV * kHD * 2, 256);
    L.total_f16 = o;
    return L;
}

// Header words at the start of the workspace.
struct PlanHeader {
    int status;     // device-side status (0 = ok)
    int n_items;    // work items in the plan (x4 KV groups = work units)
    int counter;    // dynamic work-unit counter of the attention kernel
    int pad[61];
};

// Power-of-two pre-scale applied to normalised Q/K before they are rounded to
// FP16.  After RMSNorm every entry satisfies |x_c / rms(x)| <= sqrt(128), so a
// normalised, rotated entry is bounded by sqrt(128) * max|w|.  The exponent
// is the largest e with that bound * 2^e <= 2^14, which keeps FP16 far from
// overflow for any weights; the attention logit is rescaled by 2^-(eq+ek)
// exactly.
__device__ __forceinline__ int prescale_exponent(float max_abs_w) {
    if (!(max_abs_w > 0.f)) return 0;
    float bound = max_abs_w * 11.3137084989847604f;  // sqrt(128)
    int ex;
    frexpf(16384.f / bound, &ex);                     // 16384/bound in [2^(ex-1), 2^ex)
    int e = ex - 1;
    e = e < -60 ? -60 : (e > 60 ? 60 : e);
    return e;
}

// Warp-wide max |w| over a 128-entry weight vector.
__device__ __forceinline__ float warp_max_abs128(const float* w) {
    const int lane = threadIdx.x & 31;
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) m = fmaxf(m, fabsf(w[lane + 32 * i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

// Rotation angle of NeoX RoPE for integer position `pos` and pair index f
// (0..63), inverse frequency theta^(-f/64) given in double, reduced to
// [-pi, pi] in double so large positions (up to 2^31) keep full accuracy,
// then evaluated in FP32.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
    const double two_pi_hi = 6.283185307179586;        // nearest double to 2*pi
    const double two_pi_lo = 2.4492935982947064e-16;   // 2*pi - two_pi_hi
    double a = (double)pos * inv_freq;
    double k = rint(a * 0.15915494309189535);          // a / (2*pi)
    double r = fma(-k, two_pi_hi, a);
    r = fma(-k, two_pi_lo, r);
    __sincosf((float)r, s, c);
}

// Warps per token in the preparation kernel: a call of at most 2,048 tokens
// that also prepares queries gives each token 1 + 8 warps (its keys, then
// its query heads four at a time), so that enough loads are in flight; one
// warp per token otherwise.
__host__ __device__ inline int prep_parts(int T, bool queries) {
    return (queries && T <= 2048) ? 1 + kHQ / kHKV : 1;
}

// Stages of one forward call (host side).
enum Stage : int {
    kStagePrepare = 1, kStageAttend = 2, kStageBoth = 3,
    kStageKeysReady = 4,  // with kStagePrepare: the keys were prepared by the projection GEMM
    kStageF16 = 8,        // FP16 attention-compute policy: FP32 q/k/v in, FP16 out
    kStageTileQ = 16      // prepare the queries on tile load even on sliding layers
};

// Kernel parameter blocks (passed by value).
struct PrepParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const float* q_norm_w;
    const float* k_norm_w;
    const float* sinks;
    const int* pos_ids;
    const int* cu_seqlens;
    const uint8_t* pad_mask;
    __nv_bfloat16* out;
    float* lse;
    char* ws;
    int T, nseg, batch, seqlen, window, use_rope, mode;
    int keys_ready;      // 1: the key operand is already in the workspace
    int ng;              // KV heads in the tensors (4, or a head slice of 1 or 2)
    int qprep;           // 1: normalise and rotate the queries here, FP16 into
                         // the output rows of their token (the attention kernel
                         // reads them back before writing the result there)
    int f16;             // FP16 policy: q, k, v are FP32 (qf, kf, vf); queries
                         // and values are prepared into the workspace in FP16
    const float* qf;
    const float* kf;
    const float* vf;
    float rope_theta, eps;
};

struct AttnParams {
    const float* q_norm_w;
    const float* k_norm_w;
    const float* sinks;
    const int* pos_ids;
    __nv_bfloat16* out;
    float* lse;
    char* ws;
    int T, nseg, window, use_rope;
    int ng;              // KV heads in the tensors (4, or a head slice of 1 or 2)
    float rope_theta, eps;
    // > 0: test hook.  The MMA warp of every CTA first waits this many
    // nanoseconds on a barrier nothing arrives on, so the bounded-wait
    // timeout path (status FLINT_ERR_TIMEOUT, abort, drain) runs.
    unsigned long long test_wait_ns;
};

}  // namespace flint
