// Projection GEMMs of the Flint attention layer on sm_100a (tcgen05 + TMEM +
// TMA): the fused q/k/v projection in front of the attention core and o_proj
// behind it (FlintAttention.forward on the NeMo AutoModel "flint.layers" API
// page; bias-free, FlintConfig.attention_bias = False).
//
//   D[M, N] = A[M, K] B[N, K]^T,  A, B BF16 with K contiguous (PyTorch Linear
//   weights are [out_features, in_features]), FP32 accumulation in TMEM.
//
// Epilogues:
//   plain  D -> BF16 [M, N]                                     (o_proj)
//   qkv    N = 4096 + 512 + 512: columns go to q [M, 32, 128], k [M, 4, 128]
//          and v [M, 4, 128] in BF16; for the key columns it also writes the
//          attention kernel's key operand: per-head weight-form RMSNorm with
//          k_norm_w, NeoX RoPE at the token's document-local position on
//          sliding layers, x 2^ek, FP16 [M, 4, 128] (the same arithmetic as
//          the preparation kernel's key pass, from the FP32 accumulator).
//
// Layout of one CTA (persistent, one per SM, 256 threads):
//   warp 0      TMA producer: A tile 128 x 64 and B tile 256 x 64 per stage,
//               4 stages, 128-byte swizzle
//   warp 1      TMEM owner (512 columns: two 128 x 256 FP32 accumulators);
//               lane 0 issues the MMAs (M = 128, N = 256, K = 16)
//   warps 2-3   idle
//   warps 4-7   epilogue, one thread per accumulator row (TMEM lane); each
//               warp stages 32 rows x 64 columns and stores them by TMA
// The accumulators are double-buffered, so a tile's epilogue overlaps the
// next tile's main loop.  Tiles are ordered with N fastest, so consecutive
// CTAs share an A row block in L2.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include "flint_common.cuh"
#include "sm100.cuh"

namespace flint {

constexpr int kGThreads = 256;
constexpr int kGBM = 128, kGBN = 256, kGBK = 64, kGStages = 4;
constexpr uint32_t kGABytes = kGBM * kGBK * 2;                 // 16 KiB
constexpr uint32_t kGBBytes = kGBN * kGBK * 2;                 // 32 KiB
constexpr uint32_t kGStageBytes = kGABytes + kGBBytes;
constexpr uint32_t kGOffStg = kGStages * kGStageBytes;         // 192 KiB
constexpr uint32_t kGStgBytes = 32 * 128;                      // 32 rows x 64 BF16, per epilogue warp
constexpr uint32_t kGOffBar = kGOffStg + 4 * kGStgBytes;
constexpr uint32_t kGOffMisc = kGOffBar + 16 * 8;
constexpr uint32_t kGOffInvFreq = kGOffMisc + 64;              // 64 RoPE inverse frequencies
constexpr uint32_t kGSmemUsed = kGOffInvFreq + 64 * 8;
constexpr uint32_t kGSmemBytes = kGSmemUsed + 1024;
static_assert(kGSmemBytes <= 232448, "shared memory per block");

enum : uint32_t { G_FULL = 0, G_EMPTY = 4, G_ACC_FULL = 8, G_ACC_EMPTY = 10, G_DRAIN = 12 };

enum GemmMode : int { kGemmPlain = 0, kGemmQkv = 1 };

// Column split of the fused q/k/v projection.
constexpr int kQCols = kHQ * kHD;           // 4096
constexpr int kKCols = kHKV * kHD;          // 512
constexpr int kQkvCols = kQCols + 2 * kKCols;

struct GemmParams {
    int M, N, K, mode;
    // qkv epilogue: the key operand of the attention kernel (may be null)
    __half* kn;
    const float* k_norm_w;
    float eps, rope_theta;
    int use_rope;
    // positions: pos_ids, or the index within the document / batch row
    const int* pos_ids;
    const int* cu_seqlens;   // THD boundaries (nseg + 1) or null
    int nseg, seqlen;        // seqlen > 0: rows of a [B, seqlen] mask
    int* status;             // device status word (timeouts), may be null
};

struct GMisc {
    uint32_t tmem_base;
    int abort_flag;
    float kscale;            // 2^ek
};

__device__ __forceinline__ int key_position(const GemmParams& p, int m) {
    if (p.pos_ids) return p.pos_ids[m];
    if (p.cu_seqlens) {
        int lo = 0, hi = p.nseg - 1;        // last d with cu[d] <= m
        if (hi < 0 || m >= p.cu_seqlens[p.nseg]) return 0;   // padding: unused
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.cu_seqlens[mid] <= m) lo = mid; else hi = mid - 1;
        }
        return m - p.cu_seqlens[lo];
    }
    if (p.seqlen > 0) return m % p.seqlen;
    return m;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__global__ void __launch_bounds__(kGThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
            const __grid_constant__ CUtensorMap tm_c0, const __grid_constant__ CUtensorMap tm_c1,
            const __grid_constant__ CUtensorMap tm_c2, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kGOffBar;
    auto bar = [&](uint32_t i) { return bar0 + 8u * i; };
    GMisc* misc = reinterpret_cast<GMisc*>(smem + kGOffMisc);
    volatile int* abort_flag = &misc->abort_flag;
    int* status = p.status;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int n_m = (p.M + kGBM - 1) / kGBM, n_n = (p.N + kGBN - 1) / kGBN;
    const int n_tiles = n_m * n_n, n_kb = p.K / kGBK;

    if (tid == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(bar(G_FULL + s), 1);
            mbar_init(bar(G_EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(G_ACC_FULL + a), 1);
            mbar_init(bar(G_ACC_EMPTY + a), 128);   // every epilogue thread
        }
        mbar_init(bar(G_DRAIN), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&misc->tmem_base), 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        const float mk = (p.mode == kGemmQkv && p.k_norm_w) ? warp_max_abs128(p.k_norm_w) : 0.f;
        if (lane == 0) misc->kscale = ldexpf(1.f, prescale_exponent(mk));
    }
    if (warp == 3 && p.mode == kGemmQkv && p.use_rope) {
        // theta^(-f/64), f < 64
        double* inv_freq = reinterpret_cast<double*>(smem + kGOffInvFreq);
        const double l2t = log2((double)p.rope_theta);
        inv_freq[lane] = exp2(-(double)lane / 64.0 * l2t);
        inv_freq[lane + 32] = exp2(-(double)(lane + 32) / 64.0 * l2t);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            uint32_t stage = 0, ph = 0, narmed = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                const int mt = tile / n_n, nt = tile % n_n;
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(bar(G_EMPTY + stage), ph ^ 1, abort_flag, status)) { ok = false; break; }
                    const uint32_t dst = sbase + stage * kGStageBytes;
                    mbar_expect_tx(bar(G_FULL + stage), kGStageBytes);
                    tma_load_2d(dst, &tm_a, bar(G_FULL + stage), kb * kGBK, mt * kGBM);
                    tma_load_2d(dst + kGABytes, &tm_b, bar(G_FULL + stage), kb * kGBK, nt * kGBN);
                    ++narmed;
                    if (++stage == kGStages) { stage = 0; ph ^= 1; }
                }
            }
            // drain: every armed load has landed before shared memory is released
            volatile int never = 0;
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            for (uint32_t s = 0; s < (uint32_t)kGStages; ++s) {
                // stage s received loads number s, s + 4, s + 8, ...
                if (narmed > s) {
                    const uint32_t n = (narmed - 1 - s) / kGStages + 1;
                    mbar_wait(bar(G_FULL + s), (n - 1) & 1, &never, nullptr, lim);
                }
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_f16(1, 1, 0, kGBN);
            const uint64_t da = smem_desc_sw128(sbase, 16, 1024);
            const uint64_t db = smem_desc_sw128(sbase + kGABytes, 16, 1024);
            const uint32_t a_lo = (uint32_t)da, a_hi = (uint32_t)(da >> 32);
            const uint32_t b_lo = (uint32_t)db, b_hi = (uint32_t)(db >> 32);
            uint32_t stage = 0, ph = 0, acc = 0, aph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(bar(G_ACC_EMPTY + acc), aph ^ 1, abort_flag, status)) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * kGBN;
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(bar(G_FULL + stage), ph, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t so = (stage * kGStageBytes) >> 4;
#pragma unroll
                    for (uint32_t kk = 0; kk < kGBK / 16; ++kk)
                        mma_ss_w(d, a_lo + so + kk * 2, a_hi, b_lo + so + kk * 2, b_hi, idesc,
                                 (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(G_EMPTY + stage));
                    if (++stage == kGStages) { stage = 0; ph ^= 1; }
                }
                if (!ok) break;
                mma_commit(bar(G_ACC_FULL + acc));
                acc ^= 1;
                if (acc == 0) aph ^= 1;
            }
            mma_commit(bar(G_DRAIN));
            volatile int never = 0;
            mbar_wait(bar(G_DRAIN), 0, &never, nullptr, 100ull * 1000ull * 1000ull);
        }
    } else if (warp >= 4) {
        // ================================================================ epilogue
        const int wq = warp & 3;
        const int r = 32 * wq + lane;                   // accumulator row = TMEM lane
        const uint32_t lane_base = (uint32_t)wq * 32u;
        uint8_t* stg = smem + kGOffStg + wq * kGStgBytes;
        const uint32_t stg_s = sbase + kGOffStg + wq * kGStgBytes;
        const int sw = lane & 7;
        uint32_t acc = 0, aph = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const int mt = tile / n_n, nt = tile % n_n;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(G_ACC_FULL + acc), aph, abort_flag, status))) break;
            tc_fence_after();
            const uint32_t t_acc = tmem + (lane_base << 16) + acc * kGBN;
            const int m = mt * kGBM + r;
            const int n0 = nt * kGBN;
            // destination of each 64-column block of this tile
            const CUtensorMap* map = &tm_c0;
            int col0 = n0;
            bool keys = false;
            if (p.mode == kGemmQkv) {
                if (n0 >= kQCols + kKCols) { map = &tm_c2; col0 = n0 - kQCols - kKCols; }
                else if (n0 >= kQCols) { map = &tm_c1; col0 = n0 - kQCols; keys = p.kn != nullptr; }
            }
            float ss0 = 0.f, ss1 = 0.f;                 // sum of squares of the tile's two key heads
#pragma unroll 1
            for (int j = 0; j < kGBN / 64; ++j) {
                if (n0 + 64 * j >= p.N) break;
                uint32_t v[64];
                tmem_ld32(t_acc + 64u * j, v);
                tmem_ld32(t_acc + 64u * j + 32u, v + 32);
                tmem_wait_ld();
                if (keys) {
                    float sj = 0.f;
#pragma unroll
                    for (int e = 0; e < 64; ++e) sj = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), sj);
                    if (j < 2) ss0 += sj; else ss1 += sj;
                }
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                // the staging block is free once lane 0's earlier stores have read it
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ sw) << 4)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(map, stg_s, col0 + 64 * j, mt * kGBM + 32 * wq);
                    bulk_commit_group();
                }
            }
            if (keys) {
                // the attention kernel's key operand: RMSNorm (weight form),
                // RoPE on sliding layers, x 2^ek, FP16; channel f pairs with
                // f + 64, 32 channel pairs per step.  Warp-uniform (the TMEM
                // loads are warp-collective): rows past M only skip their
                // position read and their stores.
                const bool row_ok = m < p.M;
                const float kscale = misc->kscale;
                const int hk0 = col0 / kHD;              // first key head of the tile
                const int pos = (p.use_rope && row_ok) ? key_position(p, m) : 0;
                const double* inv_freq = reinterpret_cast<const double*>(smem + kGOffInvFreq);
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    float cs[32], sn[32];
                    if (p.use_rope) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) rope_cos_sin(pos, inv_freq[32 * c + e], &cs[e], &sn[e]);
                    }
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        const float rn = rsqrtf((hh ? ss1 : ss0) * (1.f / kHD) + p.eps) * kscale;
                        uint32_t a[32], b[32];
                        tmem_ld32(t_acc + 128u * hh + 32u * c, a);
                        tmem_ld32(t_acc + 128u * hh + 64u + 32u * c, b);
                        tmem_wait_ld();
                        uint32_t ha[16], hb[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float y[2][2];
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const int f = 32 * c + e + q;
                                float n0 = __uint_as_float(a[e + q]) * rn * p.k_norm_w[f];
                                float n1 = __uint_as_float(b[e + q]) * rn * p.k_norm_w[64 + f];
                                if (p.use_rope) {
                                    const float y0 = n0 * cs[e + q] - n1 * sn[e + q];
                                    const float y1 = n1 * cs[e + q] + n0 * sn[e + q];
                                    n0 = y0; n1 = y1;
                                }
                                y[0][q] = n0; y[1][q] = n1;
                            }
                            const __half2 lo = __floats2half2_rn(y[0][0], y[0][1]);
                            const __half2 hi = __floats2half2_rn(y[1][0], y[1][1]);
                            ha[e >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
                            hb[e >> 1] = *reinterpret_cast<const uint32_t*>(&hi);
                        }
                        if (row_ok) {
                            __half* dst = p.kn + ((size_t)m * kHKV + hk0 + hh) * kHD;
                            uint4* da = reinterpret_cast<uint4*>(dst + 32 * c);
                            uint4* db = reinterpret_cast<uint4*>(dst + 64 + 32 * c);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                da[q] = make_uint4(ha[4 * q], ha[4 * q + 1], ha[4 * q + 2], ha[4 * q + 3]);
                                db[q] = make_uint4(hb[4 * q], hb[4 * q + 1], hb[4 * q + 2], hb[4 * q + 3]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(G_ACC_EMPTY + acc));
            acc ^= 1;
            if (acc == 0) aph ^= 1;
        }
        if (lane == 0) bulk_wait_group0();
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

extern const unsigned kGemmSmemBytes = kGSmemBytes;
extern const unsigned kGemmThreads = kGThreads;

}  // namespace flint

// ==================================================================== host side
#include <cuda_runtime.h>
#include "flint_host.cuh"

namespace flint {

namespace {

// 2-D map over a row-major [rows, cols] matrix of 16-bit elements: dims
// (cols, rows), box (64, box_rows), 128-byte swizzle, zero fill outside.
flint_status_t make_map2d(EncodeTiledFn enc, CUtensorMap* m, CUtensorMapDataType dt, const void* base,
                          int rows, int cols, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return FLINT_OK;
}

bool g_gemm_attr[64] = {false};

}  // namespace

__global__ void gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                            const __grid_constant__ CUtensorMap tm_c0, const __grid_constant__ CUtensorMap tm_c1,
                            const __grid_constant__ CUtensorMap tm_c2, const GemmParams p);

// Enqueues D = A B^T.  A [M, K] and B [N, K] BF16; K a multiple of 64.
// Plain mode: c0 = D [M, N] BF16, N a multiple of 64.  Qkv mode (N = 5120):
// c0 = q [M, 4096], c1 = k [M, 512], c2 = v [M, 512], p.kn optional.
flint_status_t launch_gemm(const void* a, const void* b, void* c0, void* c1, void* c2, GemmParams p,
                           cudaStream_t s) {
    int sms = 0;
    flint_status_t st = device_setup(&sms);
    if (st != FLINT_OK) return st;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return fail(FLINT_ERR_UNSUPPORTED, "device index %d", dev);
    if (!g_gemm_attr[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kGSmemBytes);
        if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        g_gemm_attr[dev] = true;
    }
    EncodeTiledFn enc = nullptr;
    st = get_encoder(&enc);
    if (st != FLINT_OK) return st;
    CUtensorMap ta, tb, t0, t1, t2;
    st = make_map2d(enc, &ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, p.M, p.K, kGBM);
    if (st != FLINT_OK) return st;
    st = make_map2d(enc, &tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, p.N, p.K, kGBN);
    if (st != FLINT_OK) return st;
    if (p.mode == kGemmQkv) {
        st = make_map2d(enc, &t0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c0, p.M, kQCols, 32);
        if (st == FLINT_OK) st = make_map2d(enc, &t1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c1, p.M, kKCols, 32);
        if (st == FLINT_OK) st = make_map2d(enc, &t2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c2, p.M, kKCols, 32);
    } else {
        st = make_map2d(enc, &t0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c0, p.M, p.N, 32);
        t1 = t0;
        t2 = t0;
    }
    if (st != FLINT_OK) return st;
    const int n_tiles = ((p.M + kGBM - 1) / kGBM) * ((p.N + kGBN - 1) / kGBN);
    const int grid = n_tiles < sms ? n_tiles : sms;
    gemm_kernel<<<grid, kGThreads, kGSmemBytes, s>>>(ta, tb, t0, t1, t2, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(e));
    return FLINT_OK;
}

flint_status_t launch_qkv_gemm(const void* x, const void* w_qkv, int T, int hidden, void* q, void* k,
                               void* v, void* kn, const float* k_norm_w, float eps, int use_rope,
                               float rope_theta, const int32_t* pos_ids, const int32_t* cu_seqlens,
                               int nseg, int seqlen, int* status, cudaStream_t s) {
    GemmParams p = {};
    p.M = T;
    p.N = kQkvCols;
    p.K = hidden;
    p.mode = kGemmQkv;
    p.kn = static_cast<__half*>(kn);
    p.k_norm_w = k_norm_w;
    p.eps = eps;
    p.rope_theta = rope_theta;
    p.use_rope = use_rope;
    p.pos_ids = pos_ids;
    p.cu_seqlens = cu_seqlens;
    p.nseg = nseg;
    p.seqlen = seqlen;
    p.status = status;
    return launch_gemm(x, w_qkv, q, k, v, p, s);
}

flint_status_t launch_plain_gemm(const void* a, const void* b, int M, int N, int K, void* c, int* status,
                                 cudaStream_t s) {
    GemmParams p = {};
    p.M = M;
    p.N = N;
    p.K = K;
    p.mode = kGemmPlain;
    p.status = status;
    return launch_gemm(a, b, c, nullptr, nullptr, p, s);
}

}  // namespace flint
