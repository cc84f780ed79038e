// Gradient of the sink-aware GQA attention forward (sm_100a, CUDA cores,
// FP32 throughout; a first correct version, not yet on the tensor cores).
//
// The pages make every head's sink a trainable FP32 parameter ("flint" model
// page on NeMo AutoModel, "Parallelism and backends": the sink adjoint, and
// FA4 rejecting learned sinks in backward).  The gradient is the exact
// derivative of the forward (FlintAttention.forward on the "flint.layers" API
// page; the sink as a zero-value softmax column, HF discussion #26 on
// RecursiveSI/flint) for a loss on `out`:
//
//   D_i   = dO_i . out_i
//   P_ij  = exp(s_ij - lse_i),  s_ij = q~_i . k~_j / sqrt(128)
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dq~_i = sum_j dS_ij k~_j / sqrt(128)      dk~_j = sum_{h,i} dS_ij q~_i / sqrt(128)
//   dv_j  = sum_{h,i} P_ij dO_i               dsink_h = -sum_i exp(sink_h - lse_i) D_i
//
// then back through RoPE (rotation by -p) and RMSNorm (weight form):
//   dw += dn * x r,   dx = r w dn - x r^3 (sum_c w_c dn_c x_c) / 128.
//
// Kernels, in stream order:
//   bwd_segments_kernel  document bounds of every token (THD boundaries or a
//                        trailing-padding mask), validated
//   bwd_prep_kernel      q~, k~ in FP32 and D per (token, head)
//   bwd_dq_kernel        a warp per (query token, 4 query heads of a KV
//                        head): loops over the token's keys
//   bwd_dkv_kernel       a warp pair per (key token, KV head), 4 query heads
//                        per warp: loops over the key's queries
//   bwd_finish_kernel    sums the per-CTA partials of dq_norm_w, dk_norm_w
//                        and dsinks in a fixed order (deterministic)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "../../include/flint_attn.h"
#include "flint_common.cuh"

namespace flint {

constexpr int kBwdThreads = 256;            // 8 warps: the query heads of one KV head
constexpr int kBwdMaxBlocks = 2048;         // grid cap; sizes the partial-sum arrays
constexpr int kBwdPartQ = kHD + kHQ;        // per-CTA partial: dq_norm_w[128], dsinks[32]
constexpr int kBwdSegThreads = 1024;

struct BwdLayout {
    size_t seg_lo, seg_hi, delta, qt, kt, part_q, part_k, total;
};

inline BwdLayout bwd_layout(int T) {
    BwdLayout L;
    size_t o = 256;                                                   // status word
    L.seg_lo = o; o = ws_align(o + sizeof(int) * (size_t)T, 256);
    L.seg_hi = o; o = ws_align(o + sizeof(int) * (size_t)T, 256);
    L.delta = o;  o = ws_align(o + sizeof(float) * (size_t)T * kHQ, 256);
    L.qt = o;     o = ws_align(o + sizeof(float) * (size_t)T * kHQ * kHD, 256);
    L.kt = o;     o = ws_align(o + sizeof(float) * (size_t)T * kHKV * kHD, 256);
    L.part_q = o; o = ws_align(o + sizeof(float) * (size_t)kBwdMaxBlocks * kBwdPartQ, 256);
    L.part_k = o; o = ws_align(o + sizeof(float) * (size_t)kBwdMaxBlocks * kHD, 256);
    L.total = o;
    return L;
}

struct BwdParams {
    const __nv_bfloat16* q;      // [T,32,128]
    const __nv_bfloat16* k;      // [T,4,128]
    const __nv_bfloat16* v;      // [T,4,128]
    const float* q_norm_w;
    const float* k_norm_w;
    const float* sinks;
    const int* pos_ids;
    const int* cu_seqlens;
    const uint8_t* pad_mask;
    const __nv_bfloat16* out;    // [T,4096]
    const float* lse;            // [32,T]
    const __nv_bfloat16* dout;   // [T,4096]
    float* dq;                   // [T,32,128]
    float* dk;                   // [T,4,128]
    float* dv;                   // [T,4,128]
    float* dq_norm_w;            // [128]
    float* dk_norm_w;            // [128]
    float* dsinks;               // [32]
    int* status;
    int* seg_lo;                 // [T]: first token of the token's document, -1 = padding
    int* seg_hi;                 // [T]: one past its last token
    float* delta;                // [T,32]: D
    float* qt;                   // [T,32,128]: q~
    float* kt;                   // [T,4,128]: k~
    float* part_q;               // [dq grid,160]
    float* part_k;               // [dk/dv grid,128]
    int T, nseg, batch, seqlen, window, use_rope, mode;
    float rope_theta, eps;
};

__device__ __forceinline__ float bf(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ void set_status(int* status, int code) { atomicCAS(status, 0, code); }

// ---- document bounds: one CTA per document (THD) or batch row (mask)
__global__ void __launch_bounds__(kBwdSegThreads) bwd_segments_kernel(const BwdParams p) {
    const int d = blockIdx.x;
    int a = 0, b = 0;
    if (p.mode == kMaskThd) {
        a = p.cu_seqlens[d];
        b = p.cu_seqlens[d + 1];
        if ((d == 0 && a != 0) || a < 0 || b < a || b > p.T) {
            if (threadIdx.x == 0) set_status(p.status, kStatusInvalid);
            return;
        }
    } else if (p.mode == kMaskPad) {
        const size_t row = (size_t)d * p.seqlen;
        int len = 0;
        for (int c = 0; c < p.seqlen; c += kBwdSegThreads) {
            const int pi = c + threadIdx.x;
            len += __syncthreads_count(pi < p.seqlen && p.pad_mask[row + pi] != 0);
        }
        int bad = 0;
        for (int c = 0; c < p.seqlen; c += kBwdSegThreads) {
            const int pi = c + threadIdx.x;
            bad |= __syncthreads_or(pi < p.seqlen && ((p.pad_mask[row + pi] != 0) != (pi < len)));
        }
        if (bad) {
            if (threadIdx.x == 0) set_status(p.status, kStatusUnsupported);
            return;
        }
        a = d * p.seqlen;
        b = a + len;
    } else {
        a = 0;
        b = p.T;
    }
    for (int t = a + threadIdx.x; t < b; t += kBwdSegThreads) {
        p.seg_lo[t] = a;
        p.seg_hi[t] = b;
    }
}

__device__ __forceinline__ int token_pos(const BwdParams& p, int t) {
    if (p.pos_ids) return p.pos_ids[t];
    const int lo = p.seg_lo[t];
    return lo >= 0 ? t - lo : 0;
}

// Normalise and rotate one row held by a warp: lane l owns channels
// l, l+32, l+64, l+96 (RoPE pairs (l, l+64) and (l+32, l+96)).
__device__ __forceinline__ void norm_rope(const float x[4], const float* w, float eps, bool rope, int pos,
                                          const double* inv, int lane, float y[4]) {
    const float ss = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float r = rsqrtf(ss * (1.f / kHD) + eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) y[i] = x[i] * r * w[lane + 32 * i];
    if (rope) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float c, s;
            rope_cos_sin(pos, inv[lane + 32 * i], &c, &s);
            const float a = y[i], b = y[i + 2];
            y[i] = a * c - b * s;
            y[i + 2] = b * c + a * s;
        }
    }
}

__device__ __forceinline__ void load_inv_freq(double* s_inv, float theta) {
    if (threadIdx.x < 64) s_inv[threadIdx.x] = exp2(-(double)threadIdx.x / 64.0 * log2((double)theta));
}

// ---- q~, k~ (FP32) and D: one warp per row, rows = T*32 query rows then T*4 key rows
__global__ void __launch_bounds__(kBwdThreads) bwd_prep_kernel(const BwdParams p) {
    __shared__ double s_inv[64];
    __shared__ float s_w[2][kHD];
    load_inv_freq(s_inv, p.rope_theta);
    if (threadIdx.x < kHD) {
        s_w[0][threadIdx.x] = p.q_norm_w[threadIdx.x];
        s_w[1][threadIdx.x] = p.k_norm_w[threadIdx.x];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const size_t nq = (size_t)p.T * kHQ, nrows = nq + (size_t)p.T * kHKV;
    const size_t wstride = (size_t)gridDim.x * (kBwdThreads / 32);
    for (size_t r = (size_t)blockIdx.x * (kBwdThreads / 32) + (threadIdx.x >> 5); r < nrows; r += wstride) {
        const bool is_q = r < nq;
        const size_t row = is_q ? r : r - nq;          // q row t*32+h, or k row t*4+g
        const int t = (int)(is_q ? row / kHQ : row / kHKV);
        const __nv_bfloat16* src = is_q ? p.q : p.k;
        float x[4], y[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = bf(src, row * kHD + lane + 32 * i);
        norm_rope(x, s_w[is_q ? 0 : 1], p.eps, p.use_rope != 0, token_pos(p, t), s_inv, lane, y);
        float* dst = (is_q ? p.qt : p.kt) + row * kHD;
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[lane + 32 * i] = y[i];
        if (is_q) {
            float d = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) d += bf(p.dout, row * kHD + lane + 32 * i) * bf(p.out, row * kHD + lane + 32 * i);
            d = warp_sum(d);
            if (lane == 0) p.delta[row] = d;
        }
    }
}

// exp(sink - lse) for one row: 0 for sink = -inf and for sink = +inf (whose
// rows have out = 0 whatever the sink, so no gradient reaches it)
__device__ __forceinline__ float sink_share(float sink, float lse) {
    if (isinf(sink)) return 0.f;
    return expf(sink - lse);
}

// Row layout of the dq and dk/dv loops: a warp carries 4 rows (4 query heads
// of one KV head), 8 lanes per row.  Lane l = 8 r + sub holds row r's
// channels 8 sub .. 8 sub + 7 and 64 + 8 sub .. 64 + 8 sub + 7 (16 values,
// index e), so each RoPE pair (c, c + 64) sits in one lane (e and e + 8) and
// a row's dot product needs 3 shuffle levels within its 8 lanes.
constexpr int kRowLanes = 8;

__device__ __forceinline__ int lane_ch(int sub, int e) { return (e < 8 ? 0 : 56) + 8 * sub + e; }

__device__ __forceinline__ float group_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    return x;
}

// Dot products of a row pair over a lane's 16 channels, as four independent
// partial sums each (short dependency chains), then summed over the row's 8 lanes.
__device__ __forceinline__ void dot2_16(const float a[16], const float b[16], const float c[16],
                                        const float d[16], float* ab, float* cd) {
    float x[4] = {0.f, 0.f, 0.f, 0.f}, y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        x[e & 3] = fmaf(a[e], b[e], x[e & 3]);
        y[e & 3] = fmaf(c[e], d[e], y[e & 3]);
    }
    *ab = group_sum((x[0] + x[1]) + (x[2] + x[3]));
    *cd = group_sum((y[0] + y[1]) + (y[2] + y[3]));
}

// 16 FP32 values of a row (two runs of 8 channels), 16-byte loads
__device__ __forceinline__ void load16f(const float* row, int sub, float v[16]) {
    const float4* a = reinterpret_cast<const float4*>(row + 8 * sub);
    const float4* b = reinterpret_cast<const float4*>(row + 64 + 8 * sub);
    const float4 x0 = a[0], x1 = a[1], y0 = b[0], y1 = b[1];
    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w; v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
    v[8] = y0.x; v[9] = y0.y; v[10] = y0.z; v[11] = y0.w; v[12] = y1.x; v[13] = y1.y; v[14] = y1.z; v[15] = y1.w;
}

__device__ __forceinline__ void unpack8(uint4 u, float* v) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// 16 BF16 values of a row, widened to FP32
__device__ __forceinline__ void load16h(const __nv_bfloat16* row, int sub, float v[16]) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + 8 * sub);
    const uint4 b = *reinterpret_cast<const uint4*>(row + 64 + 8 * sub);
    unpack8(a, v);
    unpack8(b, v + 8);
}

__device__ __forceinline__ void store16f(float* row, int sub, const float v[16]) {
    float4* a = reinterpret_cast<float4*>(row + 8 * sub);
    float4* b = reinterpret_cast<float4*>(row + 64 + 8 * sub);
    a[0] = make_float4(v[0], v[1], v[2], v[3]);
    a[1] = make_float4(v[4], v[5], v[6], v[7]);
    b[0] = make_float4(v[8], v[9], v[10], v[11]);
    b[1] = make_float4(v[12], v[13], v[14], v[15]);
}

// Adjoint of RMSNorm (weight form) then RoPE for one row in the 8-lane
// layout: dy (gradient of the rotated row) -> dx; adds dn * x * r to dw.
__device__ __forceinline__ void norm_rope_bwd16(const float x[16], const float* w, float eps, bool rope,
                                                int pos, const double* inv, int sub, const float dy[16],
                                                float dx[16], float dw[16]) {
    float dn[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) dn[e] = dy[e];
    if (rope) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float c, s;
            rope_cos_sin(pos, inv[8 * sub + e], &c, &s);
            const float a = dy[e], b = dy[e + 8];
            dn[e] = a * c + b * s;
            dn[e + 8] = b * c - a * s;
        }
    }
    float ss = 0.f, t = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        ss = fmaf(x[e], x[e], ss);
        t = fmaf(w[lane_ch(sub, e)] * dn[e], x[e], t);
    }
    ss = group_sum(ss);
    t = group_sum(t);
    const float r = rsqrtf(ss * (1.f / kHD) + eps);
    const float c3 = r * r * r * t * (1.f / kHD);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        dx[e] = r * w[lane_ch(sub, e)] * dn[e] - x[e] * c3;
        dw[e] = fmaf(dn[e] * x[e], r, dw[e]);
    }
}

// ---- dq: work item = (query token i, KV head g, half) -> query heads
// 8g + 4 half .. + 3, one per 8-lane row; longest rows first
__global__ void __launch_bounds__(kBwdThreads) bwd_dq_kernel(const BwdParams p) {
    __shared__ double s_inv[64];
    __shared__ float s_w[kHD];
    __shared__ float s_dsink[kBwdThreads / 32][kHQ];    // per warp: only that warp adds to its row
    __shared__ float s_dw[kBwdThreads / kRowLanes][kHD];
    load_inv_freq(s_inv, p.rope_theta);
    if (threadIdx.x < kHD) s_w[threadIdx.x] = p.q_norm_w[threadIdx.x];
    for (int t = threadIdx.x; t < (kBwdThreads / 32) * kHQ; t += kBwdThreads) (&s_dsink[0][0])[t] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = lane >> 3, sub = lane & 7;
    const float scale = 0.08838834764831845f;            // 1/sqrt(128)
    const float scale_log2e = scale * 1.4426950408889634f;
    float dw[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) dw[e] = 0.f;
    const int items = p.T * kHKV * 2;
    const int nwarps = gridDim.x * (kBwdThreads / 32);
    for (int it = blockIdx.x * (kBwdThreads / 32) + warp; it < items; it += nwarps) {
        const int i = p.T - 1 - it / (kHKV * 2), g = (it >> 1) % kHKV, half = it & 1;
        const int h = g * kGroup + half * 4 + r;
        const size_t qrow = (size_t)i * kHQ + h;
        float* dq = p.dq + qrow * kHD;
        const int seg = p.seg_lo[i];                       // same for the whole warp
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        if (seg < 0) {
            store16f(dq, sub, acc);
            continue;
        }
        const int lo = p.window > 0 ? max(seg, i - p.window + 1) : seg;
        float qt[16], dO[16];
        load16f(p.qt + qrow * kHD, sub, qt);
        load16h(p.dout + qrow * kHD, sub, dO);
        const float D = p.delta[qrow];
        const float sink = p.sinks[h];
        // a +inf sink: out = 0 and no gradient; an lse of +inf makes every P 0
        const float L = (isinf(sink) && sink > 0.f) ? INFINITY : p.lse[(size_t)h * p.T + i];
        const float Ll2 = L * 1.4426950408889634f;
#pragma unroll 2
        for (int j = lo; j <= i; ++j) {
            const size_t krow = ((size_t)j * kHKV + g) * kHD;
            float kv[16], vv[16];
            load16f(p.kt + krow, sub, kv);
            load16h(p.v + krow, sub, vv);
            float s, dp;
            dot2_16(qt, kv, dO, vv, &s, &dp);
            const float pr = exp2f(fmaf(s, scale_log2e, -Ll2));
            const float ds = pr * (dp - D);
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = fmaf(ds, kv[e], acc[e]);
        }
        // the warp's 4 rows are 4 different heads: plain adds in program order
        if (sub == 0) s_dsink[warp][h] += -sink_share(sink, L) * D;
        float x[16], dy[16], dx[16];
        load16h(p.q + qrow * kHD, sub, x);
#pragma unroll
        for (int e = 0; e < 16; ++e) dy[e] = acc[e] * scale;
        norm_rope_bwd16(x, s_w, p.eps, p.use_rope != 0, token_pos(p, i), s_inv, sub, dy, dx, dw);
        store16f(dq, sub, dx);
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) s_dw[warp * 4 + r][lane_ch(sub, e)] = dw[e];
    __syncthreads();
    float* part = p.part_q + (size_t)blockIdx.x * kBwdPartQ;
    if (threadIdx.x < kHD) {
        float s = 0.f;
        for (int k = 0; k < kBwdThreads / kRowLanes; ++k) s += s_dw[k][threadIdx.x];
        part[threadIdx.x] = s;
    } else if (threadIdx.x < kHD + kHQ) {
        float s = 0.f;
        for (int w = 0; w < kBwdThreads / 32; ++w) s += s_dsink[w][threadIdx.x - kHD];
        part[threadIdx.x] = s;
    }
}

__device__ __forceinline__ void pair_barrier(int pair) {
    asm volatile("bar.sync %0, 64;" ::"r"(1 + pair) : "memory");
}

// ---- dk, dv: work item = (key token j, KV head g), taken by a pair of warps
// (half 0: query heads 8g .. 8g+3, half 1: 8g+4 .. 8g+7), 4 pairs per CTA
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_dkv_kernel(const BwdParams p) {
    constexpr int kPairs = kBwdThreads / 64;
    __shared__ double s_inv[64];
    __shared__ float s_w[kHD];
    __shared__ float s_red[kPairs][2][2 * kHD];            // per warp: dk~ (128), dv (128)
    __shared__ float s_dw[kPairs][kHD];
    load_inv_freq(s_inv, p.rope_theta);
    if (threadIdx.x < kHD) s_w[threadIdx.x] = p.k_norm_w[threadIdx.x];
    for (int t = threadIdx.x; t < kPairs * kHD; t += kBwdThreads) (&s_dw[0][0])[t] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = lane >> 3, sub = lane & 7, pair = warp >> 1, half = warp & 1;
    const float scale = 0.08838834764831845f;
    const float scale_log2e = scale * 1.4426950408889634f;
    const int items = p.T * kHKV;
    for (int it = blockIdx.x * kPairs + pair; it < items; it += gridDim.x * kPairs) {
        const int j = it / kHKV, g = it % kHKV;
        const int h = g * kGroup + half * 4 + r;
        const size_t krow = (size_t)j * kHKV + g;
        const int seg = p.seg_lo[j];                        // same for both warps of the pair
        if (seg < 0) {
            if (half == 0 && r == 0) {
                float z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) z[e] = 0.f;
                store16f(p.dk + krow * kHD, sub, z);
                store16f(p.dv + krow * kHD, sub, z);
            }
            continue;
        }
        const int hi = p.window > 0 ? (int)min((long long)p.seg_hi[j], (long long)j + p.window)
                                    : p.seg_hi[j];
        float kv[16], vv[16], dk[16], dv[16];
        load16f(p.kt + krow * kHD, sub, kv);
        load16h(p.v + krow * kHD, sub, vv);
#pragma unroll
        for (int e = 0; e < 16; ++e) { dk[e] = 0.f; dv[e] = 0.f; }
        const float sink = p.sinks[h];
        const bool dead = isinf(sink) && sink > 0.f;        // +inf sink: every P is 0
        for (int i = j; i < hi; ++i) {
            const size_t qrow = (size_t)i * kHQ + h;
            float qt[16], dO[16];
            load16f(p.qt + qrow * kHD, sub, qt);
            load16h(p.dout + qrow * kHD, sub, dO);
            const float L = dead ? INFINITY : p.lse[(size_t)h * p.T + i];
            const float D = p.delta[qrow];
            float s, dp;
            dot2_16(qt, kv, dO, vv, &s, &dp);
            const float pr = exp2f(fmaf(s, scale_log2e, -L * 1.4426950408889634f));
            const float ds = pr * (dp - D);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                dk[e] = fmaf(ds, qt[e], dk[e]);
                dv[e] = fmaf(pr, dO[e], dv[e]);
            }
        }
        // sum the warp's 4 rows (lane bits 3 and 4), then the pair's 2 warps
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            dk[e] += __shfl_xor_sync(0xffffffffu, dk[e], 8);
            dk[e] += __shfl_xor_sync(0xffffffffu, dk[e], 16);
            dv[e] += __shfl_xor_sync(0xffffffffu, dv[e], 8);
            dv[e] += __shfl_xor_sync(0xffffffffu, dv[e], 16);
        }
        if (r == 0) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                s_red[pair][half][lane_ch(sub, e)] = dk[e];
                s_red[pair][half][kHD + lane_ch(sub, e)] = dv[e];
            }
        }
        pair_barrier(pair);
        if (half == 0) {
            // every row group of warp 0 computes the key's adjoint (the
            // shuffles need the whole warp); row group 0 writes the results
            // and adds the key's k_norm_w share to the pair's row of s_dw
            if (r == 0) {
                float dvs[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    dvs[e] = s_red[pair][0][kHD + lane_ch(sub, e)] + s_red[pair][1][kHD + lane_ch(sub, e)];
                store16f(p.dv + krow * kHD, sub, dvs);
            }
            float dy[16], x[16], dx[16], dw[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                dy[e] = (s_red[pair][0][lane_ch(sub, e)] + s_red[pair][1][lane_ch(sub, e)]) * scale;
                dw[e] = 0.f;
            }
            load16h(p.k + krow * kHD, sub, x);
            norm_rope_bwd16(x, s_w, p.eps, p.use_rope != 0, token_pos(p, j), s_inv, sub, dy, dx, dw);
            if (r == 0) {
                store16f(p.dk + krow * kHD, sub, dx);
#pragma unroll
                for (int e = 0; e < 16; ++e) s_dw[pair][lane_ch(sub, e)] += dw[e];
            }
        }
        pair_barrier(pair);                                 // s_red is free for the next item
    }
    __syncthreads();
    if (threadIdx.x < kHD) {
        float s = 0.f;
        for (int k = 0; k < kPairs; ++k) s += s_dw[k][threadIdx.x];
        p.part_k[(size_t)blockIdx.x * kHD + threadIdx.x] = s;
    }
}

// ---- fixed-order sums of the per-CTA partials
__global__ void bwd_finish_kernel(const BwdParams p, int grid_q, int grid_k) {
    const int t = threadIdx.x;
    if (t < kHD) {
        float sq = 0.f, sk = 0.f;
        for (int b = 0; b < grid_q; ++b) sq += p.part_q[(size_t)b * kBwdPartQ + t];
        for (int b = 0; b < grid_k; ++b) sk += p.part_k[(size_t)b * kHD + t];
        p.dq_norm_w[t] = sq;
        p.dk_norm_w[t] = sk;
    } else if (t < kHD + kHQ) {
        float s = 0.f;
        for (int b = 0; b < grid_q; ++b) s += p.part_q[(size_t)b * kBwdPartQ + t];
        p.dsinks[t - kHD] = s;
    }
}

flint_status_t set_error(flint_status_t s, const char* msg);

size_t bwd_workspace_bytes(int T) { return bwd_layout(T).total; }

flint_status_t run_bwd(const void* q, const void* k, const void* v, const float* q_norm_w,
                       const float* k_norm_w, const float* sinks, const int32_t* pos_ids,
                       const int32_t* cu_seqlens, int32_t num_docs, const uint8_t* pad_mask,
                       int32_t batch, int32_t seqlen, int32_t T, int32_t window, int32_t use_rope,
                       float rope_theta, float eps, const void* out, const float* lse, const void* dout,
                       float* dq, float* dk, float* dv, float* dq_norm_w, float* dk_norm_w,
                       float* dsinks, void* workspace, int sms, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    const BwdLayout L = bwd_layout(T);
    BwdParams bp;
    bp.q = static_cast<const __nv_bfloat16*>(q);
    bp.k = static_cast<const __nv_bfloat16*>(k);
    bp.v = static_cast<const __nv_bfloat16*>(v);
    bp.q_norm_w = q_norm_w;
    bp.k_norm_w = k_norm_w;
    bp.sinks = sinks;
    bp.pos_ids = use_rope ? pos_ids : nullptr;
    bp.cu_seqlens = cu_seqlens;
    bp.pad_mask = pad_mask;
    bp.out = static_cast<const __nv_bfloat16*>(out);
    bp.lse = lse;
    bp.dout = static_cast<const __nv_bfloat16*>(dout);
    bp.dq = dq;
    bp.dk = dk;
    bp.dv = dv;
    bp.dq_norm_w = dq_norm_w;
    bp.dk_norm_w = dk_norm_w;
    bp.dsinks = dsinks;
    bp.status = reinterpret_cast<int*>(ws);
    bp.seg_lo = reinterpret_cast<int*>(ws + L.seg_lo);
    bp.seg_hi = reinterpret_cast<int*>(ws + L.seg_hi);
    bp.delta = reinterpret_cast<float*>(ws + L.delta);
    bp.qt = reinterpret_cast<float*>(ws + L.qt);
    bp.kt = reinterpret_cast<float*>(ws + L.kt);
    bp.part_q = reinterpret_cast<float*>(ws + L.part_q);
    bp.part_k = reinterpret_cast<float*>(ws + L.part_k);
    bp.T = T;
    bp.batch = batch;
    bp.seqlen = seqlen;
    bp.window = window;
    bp.use_rope = use_rope;
    bp.rope_theta = rope_theta;
    bp.eps = eps;
    int nseg = 1;
    bp.mode = kMaskSingle;
    if (cu_seqlens) {
        bp.mode = kMaskThd;
        nseg = num_docs;
    } else if (pad_mask) {
        bp.mode = kMaskPad;
        nseg = batch;
    }
    bp.nseg = nseg;
    // dq: T x 8 warp items, 8 per CTA; dk/dv: T x 4 pair items, 4 per CTA;
    // both grids one wave of resident CTAs (capped by the partial arrays)
    int occ_q = 0, occ_k = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_q, bwd_dq_kernel, kBwdThreads, 0);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_k, bwd_dkv_kernel, kBwdThreads, 0);
    auto grid_for = [&](int occ) {
        long long g = (long long)sms * (occ > 0 ? occ : 1);
        if (g > kBwdMaxBlocks) g = kBwdMaxBlocks;
        if (g > T) g = T;
        return (int)g;
    };
    const int grid_q = grid_for(occ_q), grid_k = grid_for(occ_k);

    cudaError_t e = cudaMemsetAsync(ws, 0, 256, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(bp.seg_lo, 0xff, sizeof(int) * (size_t)T, s);
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: workspace reset failed");
    if (nseg > 0) {
        bwd_segments_kernel<<<nseg, kBwdSegThreads, 0, s>>>(bp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: segment launch failed");
    }
    const size_t rows = (size_t)T * (kHQ + kHKV);
    size_t prep_grid = (rows + kBwdThreads / 32 - 1) / (kBwdThreads / 32);
    if (prep_grid > (size_t)sms * 16) prep_grid = (size_t)sms * 16;
    bwd_prep_kernel<<<(unsigned)prep_grid, kBwdThreads, 0, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: prep launch failed");
    bwd_dq_kernel<<<grid_q, kBwdThreads, 0, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: dq launch failed");
    bwd_dkv_kernel<<<grid_k, kBwdThreads, 0, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: dk/dv launch failed");
    bwd_finish_kernel<<<1, kHD + kHQ, 0, s>>>(bp, grid_q, grid_k);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: finish launch failed");
    return FLINT_OK;
}

}  // namespace flint
