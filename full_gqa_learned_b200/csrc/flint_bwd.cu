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
//   bwd_dq_kernel        one warp per (query token, head): loops over its keys
//   bwd_dkv_kernel       one CTA per (key token, KV head), a warp per query
//                        head of the group: loops over the key's queries
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
    float* part_q;               // [grid,160]
    float* part_k;               // [grid,128]
    int T, nseg, batch, seqlen, window, use_rope, mode, grid;
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

// Adjoint of norm_rope: dy (gradient of the rotated row) -> dx; adds the
// row's contribution dn * x * r to dw[4].
__device__ __forceinline__ void norm_rope_bwd(const float x[4], const float* w, float eps, bool rope,
                                              int pos, const double* inv, int lane, const float dy[4],
                                              float dx[4], float dw[4]) {
    float dn[4] = {dy[0], dy[1], dy[2], dy[3]};
    if (rope) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float c, s;
            rope_cos_sin(pos, inv[lane + 32 * i], &c, &s);
            const float a = dy[i], b = dy[i + 2];
            dn[i] = a * c + b * s;
            dn[i + 2] = b * c - a * s;
        }
    }
    const float ss = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float r = rsqrtf(ss * (1.f / kHD) + eps);
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) t += w[lane + 32 * i] * dn[i] * x[i];
    t = warp_sum(t);
    const float c3 = r * r * r * t * (1.f / kHD);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        dx[i] = r * w[lane + 32 * i] * dn[i] - x[i] * c3;
        dw[i] += dn[i] * x[i] * r;
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

// ---- dq: unit u = (query token i, KV head g), longest rows first; warp w takes head 8g+w
__global__ void __launch_bounds__(kBwdThreads) bwd_dq_kernel(const BwdParams p) {
    __shared__ double s_inv[64];
    __shared__ float s_w[kHD];
    __shared__ float s_dsink[kHQ];
    __shared__ float s_dw[kBwdThreads / 32][kHD];
    load_inv_freq(s_inv, p.rope_theta);
    if (threadIdx.x < kHD) s_w[threadIdx.x] = p.q_norm_w[threadIdx.x];
    if (threadIdx.x < kHQ) s_dsink[threadIdx.x] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float scale = 0.08838834764831845f;            // 1/sqrt(128)
    const float scale_log2e = scale * 1.4426950408889634f;
    float dw[4] = {0.f, 0.f, 0.f, 0.f};
    const int units = p.T * kHKV;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int i = p.T - 1 - u / kHKV, g = u % kHKV, h = g * kGroup + warp;
        const size_t qrow = (size_t)i * kHQ + h;
        float* dq = p.dq + qrow * kHD;
        const int seg = p.seg_lo[i];
        if (seg < 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c) dq[lane + 32 * c] = 0.f;
            continue;
        }
        const int lo = p.window > 0 ? max(seg, i - p.window + 1) : seg;
        float qt[4], dO[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            qt[c] = p.qt[qrow * kHD + lane + 32 * c];
            dO[c] = bf(p.dout, qrow * kHD + lane + 32 * c);
        }
        const float D = p.delta[qrow];
        const float L = p.lse[(size_t)h * p.T + i];
        const float sink = p.sinks[h];
        if (!(isinf(sink) && sink > 0.f)) {
            const float Ll2 = L * 1.4426950408889634f;
            for (int j = lo; j <= i; ++j) {
                const size_t krow = ((size_t)j * kHKV + g) * kHD;
                float kv[4], vv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    kv[c] = p.kt[krow + lane + 32 * c];
                    vv[c] = bf(p.v, krow + lane + 32 * c);
                }
                float s = qt[0] * kv[0] + qt[1] * kv[1] + qt[2] * kv[2] + qt[3] * kv[3];
                float dp = dO[0] * vv[0] + dO[1] * vv[1] + dO[2] * vv[2] + dO[3] * vv[3];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    s += __shfl_xor_sync(0xffffffffu, s, o);
                    dp += __shfl_xor_sync(0xffffffffu, dp, o);
                }
                const float pr = exp2f(fmaf(s, scale_log2e, -Ll2));
                const float ds = pr * (dp - D);
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[c] = fmaf(ds, kv[c], acc[c]);
            }
            if (lane == 0) atomicAdd(&s_dsink[h], -sink_share(sink, L) * D);
        }
        float x[4], dy[4], dx[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            x[c] = bf(p.q, qrow * kHD + lane + 32 * c);
            dy[c] = acc[c] * scale;
        }
        norm_rope_bwd(x, s_w, p.eps, p.use_rope != 0, token_pos(p, i), s_inv, lane, dy, dx, dw);
#pragma unroll
        for (int c = 0; c < 4; ++c) dq[lane + 32 * c] = dx[c];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) s_dw[warp][lane + 32 * c] = dw[c];
    __syncthreads();
    float* part = p.part_q + (size_t)blockIdx.x * kBwdPartQ;
    if (threadIdx.x < kHD) {
        float s = 0.f;
        for (int w = 0; w < kBwdThreads / 32; ++w) s += s_dw[w][threadIdx.x];
        part[threadIdx.x] = s;
    } else if (threadIdx.x < kHD + kHQ) {
        part[threadIdx.x] = s_dsink[threadIdx.x - kHD];
    }
}

// ---- dk, dv: unit u = (key token j, KV head g); warp w takes query head 8g+w
__global__ void __launch_bounds__(kBwdThreads) bwd_dkv_kernel(const BwdParams p) {
    __shared__ double s_inv[64];
    __shared__ float s_w[kHD];
    __shared__ float s_red[kBwdThreads / 32][2 * kHD];
    load_inv_freq(s_inv, p.rope_theta);
    if (threadIdx.x < kHD) s_w[threadIdx.x] = p.k_norm_w[threadIdx.x];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float scale = 0.08838834764831845f;
    const float scale_log2e = scale * 1.4426950408889634f;
    float dw[4] = {0.f, 0.f, 0.f, 0.f};                  // warp 0 only
    const int units = p.T * kHKV;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int j = u / kHKV, g = u % kHKV, h = g * kGroup + warp;
        const size_t krow = (size_t)j * kHKV + g;
        const int seg = p.seg_lo[j];
        __syncthreads();                                  // s_red of the previous unit is consumed
        if (seg < 0) {
            if (warp == 0) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    p.dk[krow * kHD + lane + 32 * c] = 0.f;
                    p.dv[krow * kHD + lane + 32 * c] = 0.f;
                }
            }
            continue;                                     // uniform over the CTA
        }
        const int hi = p.window > 0 ? (int)min((long long)p.seg_hi[j], (long long)j + p.window)
                                    : p.seg_hi[j];
        float kv[4], vv[4], dk[4] = {0.f, 0.f, 0.f, 0.f}, dv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            kv[c] = p.kt[krow * kHD + lane + 32 * c];
            vv[c] = bf(p.v, krow * kHD + lane + 32 * c);
        }
        const float sink = p.sinks[h];
        if (!(isinf(sink) && sink > 0.f)) {
            for (int i = j; i < hi; ++i) {
                const size_t qrow = (size_t)i * kHQ + h;
                float qt[4], dO[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    qt[c] = p.qt[qrow * kHD + lane + 32 * c];
                    dO[c] = bf(p.dout, qrow * kHD + lane + 32 * c);
                }
                float s = qt[0] * kv[0] + qt[1] * kv[1] + qt[2] * kv[2] + qt[3] * kv[3];
                float dp = dO[0] * vv[0] + dO[1] * vv[1] + dO[2] * vv[2] + dO[3] * vv[3];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    s += __shfl_xor_sync(0xffffffffu, s, o);
                    dp += __shfl_xor_sync(0xffffffffu, dp, o);
                }
                const float L = p.lse[(size_t)h * p.T + i];
                const float pr = exp2f(fmaf(s, scale_log2e, -L * 1.4426950408889634f));
                const float ds = pr * (dp - p.delta[qrow]);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    dk[c] = fmaf(ds, qt[c], dk[c]);
                    dv[c] = fmaf(pr, dO[c], dv[c]);
                }
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            s_red[warp][lane + 32 * c] = dk[c];
            s_red[warp][kHD + lane + 32 * c] = dv[c];
        }
        __syncthreads();
        if (warp == 0) {
            float dy[4], x[4], dx[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float sk = 0.f, sv = 0.f;
                for (int w = 0; w < kBwdThreads / 32; ++w) {
                    sk += s_red[w][lane + 32 * c];
                    sv += s_red[w][kHD + lane + 32 * c];
                }
                dy[c] = sk * scale;
                p.dv[krow * kHD + lane + 32 * c] = sv;
                x[c] = bf(p.k, krow * kHD + lane + 32 * c);
            }
            norm_rope_bwd(x, s_w, p.eps, p.use_rope != 0, token_pos(p, j), s_inv, lane, dy, dx, dw);
#pragma unroll
            for (int c = 0; c < 4; ++c) p.dk[krow * kHD + lane + 32 * c] = dx[c];
        }
    }
    if (warp == 0) {
        float* part = p.part_k + (size_t)blockIdx.x * kHD;
#pragma unroll
        for (int c = 0; c < 4; ++c) part[lane + 32 * c] = dw[c];
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
    const int units = T * kHKV;
    int grid = sms * 8;
    if (grid > kBwdMaxBlocks) grid = kBwdMaxBlocks;
    if (grid > units) grid = units;
    bp.grid = grid;

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
    bwd_dq_kernel<<<grid, kBwdThreads, 0, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: dq launch failed");
    bwd_dkv_kernel<<<grid, kBwdThreads, 0, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: dk/dv launch failed");
    bwd_finish_kernel<<<1, kHD + kHQ, 0, s>>>(bp, grid, grid);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: finish launch failed");
    return FLINT_OK;
}

}  // namespace flint
