// Tensor-core part of the gradient of the sink-aware GQA attention (sm_100a:
// tcgen05 + TMEM + TMA).  With P_ij = exp(s_ij - lse_i), s_ij = q~_i . k~_j /
// sqrt(128), D_i = dO_i . out_i and dS_ij = P_ij (dO_i . v_j - D_i):
//
//   dq~_i = sum_j dS_ij k~_j / sqrt(128)          (bwd_dq_tc_kernel)
//   dk~_j = sum_{h,i} dS_ij q~_i / sqrt(128)      (bwd_dkv_tc_kernel)
//   dv_j  = sum_{h,i} P_ij dO_i                    (bwd_dkv_tc_kernel)
//
// (the gradient of the forward on the "flint.layers" API page of NeMo
// AutoModel, FlintAttention.forward, with the learned sink as a zero-value
// softmax column: HF discussion #26 on RecursiveSI/flint; the sink itself and
// the RoPE / RMSNorm adjoints are handled by the CUDA-core kernels around
// these two).  Operands, as in the forward: q~, k~ in FP16 scaled by powers of
// two (2^eq, 2^ek, undone exactly), dO and v in BF16, P in BF16 and dS in
// FP16 as the TMEM operands of the second products; FP32 accumulation.
//
// A 128-row query tile packs 16 tokens x the 8 query heads of one KV head (as
// in the forward); a key tile is 128 consecutive tokens of one KV head.  Tiles
// are taken at fixed token offsets; rows of other documents, of padding or
// beyond T are masked per element (key j is visible to query i when
// lo_i <= j <= i, lo_i the start of i's document or window).
//
//   dq kernel, per query tile, over its key chunks:
//     S = Qh Kh^T, dP = dO V^T  (SS)  ->  dS (threads)  ->  dQ += dS Kh  (TS)
//     TMEM: S 0..127 (dS over its first 64 columns), dP 128..255, dQ 256..383
//   dkv kernel, per key tile, over the query tiles that see it:
//     S^T = Kh Qh^T, dP^T = V dO^T  (SS)  ->  P^T, dS^T (threads)  ->
//     dV += P^T dO, dK += dS^T Qh  (TS)
//     On short sequences a key tile's query tiles are cut into pieces that
//     different CTAs run; each piece adds its dK, dV to the sum of the
//     pieces before it, in piece order, behind a per-tile flag.
//     TMEM: S^T 0..127 (P^T over its first 64), dP^T 128..255 (dS^T over its
//     first 64), dV 256..383, dK 384..511
// Each CTA (persistent, 256 threads): warp 0 scheduler + TMA producer, warp 1
// TMEM owner and MMA issuer, warps 4-7 one thread per TMEM lane.  Every wait
// is bounded (FLINT_ERR_TIMEOUT in the status word, then a drain).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "flint_common.cuh"
#include "flint_host.cuh"
#include "sm100.cuh"

namespace flint {

constexpr int kBtThreads = 384;
constexpr uint32_t kBtTile = 128 * kHD * 2;          // 32 KiB: 128 rows x 128 x 16-bit
constexpr uint32_t kBtHalf = kBtTile / 2;

// dq kernel shared memory: Q, dO tiles; 2 K and 2 V stages
constexpr uint32_t kDqOffQ = 0, kDqOffDo = kBtTile, kDqOffK = 2 * kBtTile, kDqOffV = 4 * kBtTile;
constexpr uint32_t kDqOffBar = 6 * kBtTile;
// dkv kernel shared memory: K, V tiles; 2 stages of (Q, dO) tiles, lse2 / D per stage
constexpr uint32_t kDkOffK = 0, kDkOffV = kBtTile, kDkOffQ = 2 * kBtTile, kDkOffDo = 4 * kBtTile;
constexpr uint32_t kDkOffCol = 6 * kBtTile;          // [2 stages][lse2 128, D 128] floats
constexpr uint32_t kDkOffBar = kDkOffCol + 2 * 256 * 4;
constexpr uint32_t kBtBars = 24;
constexpr uint32_t kBtOffMisc = 8 * kBtBars;         // after the barriers
constexpr uint32_t kBtSmemDq = kDqOffBar + kBtOffMisc + 64 + 1024;
constexpr uint32_t kBtSmemDk = kDkOffBar + kBtOffMisc + 64 + 1024;
static_assert(kBtSmemDq <= 232448 && kBtSmemDk <= 232448, "shared memory per block");

struct BwdTcParams {
    const float* q_norm_w;
    const float* k_norm_w;
    const float* lse;        // [32, T]
    const float* delta;      // [T, 32]
    const int* seg_lo;       // [T]: first token of the document, -1 = padding
    const int* seg_hi;       // [T]: one past its last token
    float* dq;               // [T, 32, 128]: dq~ on exit (valid rows)
    float* dk;               // [T, 4, 128]: dk~ on exit (valid rows)
    float* dv;               // [T, 4, 128]: dv on exit (valid rows)
    int* status;
    int* counter;            // dynamic unit counter (zeroed before the launch)
    int* flags;              // dkv: [key tile][KV head] pieces summed so far (zeroed)
    int T, window;
    int qp;                  // dkv: query tiles per piece of a key tile's range
    int np;                  // dkv: pieces per key tile at most
};

struct BtMisc {
    int sched[2][4];         // unit, and its range (start, count)
    uint32_t tmem_base;
    int abort_flag;
    int fix_ok;              // dkv: the previous piece's flag was seen
    float logit_scale;       // log2(e)/sqrt(128) 2^-(eq+ek)
    float dq_scale;          // 2^-ek / sqrt(128)
    float dk_scale;          // 2^-eq / sqrt(128)
};

enum : uint32_t {
    T_SCHED_FULL = 0, T_SCHED_EMPTY = 2,
    T_A_FULL = 4, T_A_EMPTY = 6,         // dq: K stages; dkv: (Q, dO) stages
    T_B_FULL = 8, T_B_EMPTY = 10,        // dq: V stages; dkv: (K, V) tile (index 0)
    T_C_FULL = 12, T_C_EMPTY = 13,       // dq: (Q, dO) tile
    T_S_FULL = 14, T_DS_READY = 15, T_ACC_FULL = 16, T_DRAIN = 17,
    T_GO = 18, T_FIX = 19                // dkv: piece fix-up hand-offs
};

__device__ __forceinline__ float bt_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t bt_pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t bt_pack_f16(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Key range of a query tile (tokens i0 .. i0+15): [kb, ke), or ke = kb when
// no row of the tile is a valid query.
__device__ __forceinline__ void q_tile_keys(const BwdTcParams& p, int i0, int* kb, int* ke) {
    int lo = 1 << 30, hi = -1;
    for (int d = 0; d < kTokPerTile; ++d) {
        const int i = i0 + d;
        if (i >= p.T) break;
        const int s = p.seg_lo[i];
        if (s < 0) continue;
        const int l = p.window > 0 ? max(s, i - p.window + 1) : s;
        lo = min(lo, l);
        hi = i;
    }
    *kb = hi < 0 ? 0 : lo;
    *ke = hi < 0 ? 0 : hi + 1;
}

// Query range of a key tile (tokens j0 .. j0+127): [qb, qe), or qe = qb.
__device__ __forceinline__ void k_tile_queries(const BwdTcParams& p, int j0, int* qb, int* qe) {
    int lo = 1 << 30, hi = -1;
    for (int d = 0; d < 128; ++d) {
        const int j = j0 + d;
        if (j >= p.T) break;
        if (p.seg_lo[j] < 0) continue;
        int e = p.seg_hi[j];
        if (p.window > 0) e = min(e, j + p.window);
        lo = min(lo, j);
        hi = max(hi, e);
    }
    *qb = hi < 0 ? 0 : lo;
    *qe = hi < 0 ? 0 : hi;
}

__device__ __forceinline__ void bt_setup_scales(const BwdTcParams& p, BtMisc* misc, int lane) {
    const float mq = warp_max_abs128(p.q_norm_w);
    const float mk = warp_max_abs128(p.k_norm_w);
    if (lane == 0) {
        const int eq = prescale_exponent(mq), ek = prescale_exponent(mk);
        misc->logit_scale = ldexpf(1.4426950408889634f * 0.08838834764831845f, -(eq + ek));
        misc->dq_scale = ldexpf(0.08838834764831845f, -ek);
        misc->dk_scale = ldexpf(0.08838834764831845f, -eq);
    }
}

// ============================================================================ dq
__global__ void __launch_bounds__(kBtThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_v,
                 const BwdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kDqOffBar;
    auto bar = [&](uint32_t i) { return bar0 + 8u * i; };
    BtMisc* misc = reinterpret_cast<BtMisc*>(smem + kDqOffBar + kBtOffMisc);
    volatile int* abort_flag = &misc->abort_flag;
    int* status = p.status;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tiles = (p.T + kTokPerTile - 1) / kTokPerTile;
    const int n_units = n_tiles * kHKV;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(T_SCHED_FULL + s), 1);
            mbar_init(bar(T_SCHED_EMPTY + s), 1 + 8);     // MMA thread + 8 row warps
            mbar_init(bar(T_A_FULL + s), 1);
            mbar_init(bar(T_A_EMPTY + s), 1);
            mbar_init(bar(T_B_FULL + s), 1);
            mbar_init(bar(T_B_EMPTY + s), 1);
        }
        mbar_init(bar(T_C_FULL), 1);
        mbar_init(bar(T_C_EMPTY), 1);
        mbar_init(bar(T_S_FULL), 1);
        mbar_init(bar(T_DS_READY), 256);
        mbar_init(bar(T_ACC_FULL), 1);
        mbar_init(bar(T_DRAIN), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&misc->tmem_base), 512);
        tmem_relinquish();
    }
    if (warp == 2) bt_setup_scales(p, misc, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ scheduler + producer
        if (lane == 0) {
            uint32_t sslot = 0, sph = 0, cph = 0, st = 0, ph = 0, narm_c = 0, narm = 0;
            bool ok = true;
            for (;;) {
                int u = atomicAdd(p.counter, 1);
                int kb = 0, ke = 0;
                if (u >= n_units) u = -1;
                else {
                    // longest tiles (the last tokens of a causal sequence) first
                    const int m = n_tiles - 1 - u / kHKV;
                    q_tile_keys(p, m * kTokPerTile, &kb, &ke);
                }
                if (!mbar_wait(bar(T_SCHED_EMPTY + sslot), sph ^ 1, abort_flag, status)) break;
                misc->sched[sslot][0] = u;
                misc->sched[sslot][1] = kb;
                misc->sched[sslot][2] = (ke - kb + 127) / 128;
                mbar_arrive(bar(T_SCHED_FULL + sslot));
                sslot ^= 1; if (sslot == 0) sph ^= 1;
                if (u < 0) break;
                const int nch = (ke - kb + 127) / 128;
                if (nch == 0) continue;
                const int g = u % kHKV, i0 = (n_tiles - 1 - u / kHKV) * kTokPerTile;
                ok = mbar_wait(bar(T_C_EMPTY), cph ^ 1, abort_flag, status);
                if (!ok) break;
                mbar_expect_tx(bar(T_C_FULL), 2 * kBtTile);
                tma_load_3d(sbase + kDqOffQ, &tm_qh, bar(T_C_FULL), 0, kGroup * g, i0);
                tma_load_3d(sbase + kDqOffQ + kBtHalf, &tm_qh, bar(T_C_FULL), 64, kGroup * g, i0);
                tma_load_3d(sbase + kDqOffDo, &tm_do, bar(T_C_FULL), 0, kGroup * g, i0);
                tma_load_3d(sbase + kDqOffDo + kBtHalf, &tm_do, bar(T_C_FULL), 64, kGroup * g, i0);
                ++narm_c;
                cph ^= 1;
                for (int c = 0; c < nch && ok; ++c) {
                    const int ks = kb + 128 * c;
                    ok = mbar_wait(bar(T_A_EMPTY + st), ph ^ 1, abort_flag, status);
                    if (!ok) break;
                    ok = mbar_wait(bar(T_B_EMPTY + st), ph ^ 1, abort_flag, status);
                    if (!ok) break;
                    mbar_expect_tx(bar(T_A_FULL + st), kBtTile);
                    tma_load_3d(sbase + kDqOffK + st * kBtTile, &tm_kh, bar(T_A_FULL + st), 0, g, ks);
                    tma_load_3d(sbase + kDqOffK + st * kBtTile + kBtHalf, &tm_kh, bar(T_A_FULL + st), 64, g, ks);
                    mbar_expect_tx(bar(T_B_FULL + st), kBtTile);
                    tma_load_3d(sbase + kDqOffV + st * kBtTile, &tm_v, bar(T_B_FULL + st), 0, g, ks);
                    tma_load_3d(sbase + kDqOffV + st * kBtTile + kBtHalf, &tm_v, bar(T_B_FULL + st), 64, g, ks);
                    ++narm;
                    st ^= 1; if (st == 0) ph ^= 1;
                }
                if (!ok) break;
            }
            // drain: every armed load has landed before shared memory is released
            volatile int never = 0;
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            if (narm_c) mbar_wait(bar(T_C_FULL), (narm_c - 1) & 1, &never, nullptr, lim);
            for (uint32_t s = 0; s < 2; ++s) {
                const uint32_t n = (narm + 1 - s) / 2;
                if (n) {
                    mbar_wait(bar(T_A_FULL + s), (n - 1) & 1, &never, nullptr, lim);
                    mbar_wait(bar(T_B_FULL + s), (n - 1) & 1, &never, nullptr, lim);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_f16(0, 0, 0, 128);     // FP16 x FP16, K-major B
            const uint32_t id_dp = idesc_f16(1, 1, 0, 128);    // BF16 x BF16, K-major B
            const uint32_t id_dq = idesc_f16(0, 0, 1, 128);    // FP16 dS (TMEM) x FP16 K, MN-major B
            const uint64_t dq0 = smem_desc_sw128(sbase + kDqOffQ, 16, 1024);
            const uint64_t ddo = smem_desc_sw128(sbase + kDqOffDo, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sbase + kDqOffK, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + kDqOffV, 16, 1024);
            const uint64_t dkm = smem_desc_sw128(sbase + kDqOffK, kBtHalf, 1024);
            constexpr uint32_t kStep = kBtTile >> 4;
            uint32_t sslot = 0, sph = 0, cph = 0, st = 0, ph = 0, dsph = 0;
            bool ok = true;
            for (; ok;) {
                if (!mbar_wait(bar(T_SCHED_FULL + sslot), sph, abort_flag, status)) break;
                const int u = misc->sched[sslot][0];
                const int nch = misc->sched[sslot][2];
                mbar_arrive(bar(T_SCHED_EMPTY + sslot));
                sslot ^= 1; if (sslot == 0) sph ^= 1;
                if (u < 0) break;
                if (nch == 0) continue;
                if (!mbar_wait(bar(T_C_FULL), cph, abort_flag, status)) break;
                cph ^= 1;
                for (int c = 0; c < nch; ++c) {
                    ok = mbar_wait(bar(T_A_FULL + st), ph, abort_flag, status) &&
                         mbar_wait(bar(T_B_FULL + st), ph, abort_flag, status);
                    if (!ok) break;
                    tc_fence_after();
                    // S = Qh Kh^T, dP = dO V^T (K = 128 channels, 8 steps of 16)
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * (kBtHalf >> 4) + (kk & 3) * 2;
                        mma_ss(tmem, dq0 + off, dk0 + st * kStep + off, id_s, kk > 0);
                    }
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * (kBtHalf >> 4) + (kk & 3) * 2;
                        mma_ss(tmem + 128, ddo + off, dv0 + st * kStep + off, id_dp, kk > 0);
                    }
                    mma_commit(bar(T_S_FULL));
                    mma_commit(bar(T_B_EMPTY + st));               // V chunk done
                    ok = mbar_wait(bar(T_DS_READY), dsph, abort_flag, status);
                    if (!ok) break;
                    dsph ^= 1;
                    tc_fence_after();
                    // dQ += dS Kh (K = 128 keys, 8 steps of 16; dS in TMEM:
                    // keys 0..63 in columns 0..31, keys 64..127 in 64..95)
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + 256, tmem + 8 * kk + (kk >= 4 ? 32u : 0u), dkm + st * kStep + kk * (2048 >> 4),
                               id_dq, (c > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(T_A_EMPTY + st));               // K chunk done
                    st ^= 1; if (st == 0) ph ^= 1;
                }
                if (!ok) break;
                mma_commit(bar(T_C_EMPTY));
                mma_commit(bar(T_ACC_FULL));
            }
            mma_commit(bar(T_DRAIN));
            volatile int never = 0;
            mbar_wait(bar(T_DRAIN), 0, &never, nullptr, 100ull * 1000ull * 1000ull);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ rows: dS, then dq~
        // Two warpgroups: warps 4-7 take the key columns 0..63 of every row,
        // warps 8-11 the columns 64..127; each writes its dS (FP16 pairs)
        // inside its own columns (0..31, 64..95), so neither overwrites S
        // the other has yet to read.
        const int half = (warp - 4) >> 2;
        const int r = (tid - 128) & 127;                // TMEM lane = tile row
        const int tl = r >> 3, hl = r & 7;
        const uint32_t lb = (uint32_t)(warp & 3) * 32u;
        const uint32_t t_s = tmem + (lb << 16), t_dp = t_s + 128, t_dq = t_s + 256;
        const float C = misc->logit_scale, dqs = misc->dq_scale;
        uint32_t sslot = 0, sph = 0, s_ph = 0, aph = 0;
        for (;;) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(T_SCHED_FULL + sslot), sph, abort_flag, status))) break;
            const int u = misc->sched[sslot][0];
            const int kb = misc->sched[sslot][1], nch = misc->sched[sslot][2];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(T_SCHED_EMPTY + sslot));
            sslot ^= 1; if (sslot == 0) sph ^= 1;
            if (u < 0) break;
            if (nch == 0) continue;
            const int g = u % kHKV, i0 = (n_tiles - 1 - u / kHKV) * kTokPerTile;
            const int i = i0 + tl, h = kGroup * g + hl;
            const bool valid = i < p.T && p.seg_lo[i] >= 0;
            int lo = 0;
            float lse2 = 0.f, D = 0.f;
            if (valid) {
                lo = p.window > 0 ? max(p.seg_lo[i], i - p.window + 1) : p.seg_lo[i];
                lse2 = p.lse[(size_t)h * p.T + i] * 1.4426950408889634f;
                D = p.delta[(size_t)i * kHQ + h];
            }
            bool alive = true;
            for (int c = 0; c < nch; ++c) {
                if (!__all_sync(0xffffffffu, mbar_wait(bar(T_S_FULL), s_ph, abort_flag, status))) {
                    alive = false;
                    break;
                }
                s_ph ^= 1;
                tc_fence_after();
                const int ks = kb + 128 * c;
#pragma unroll 1
                for (int b = 2 * half; b < 2 * half + 2; ++b) {
                    uint32_t sv[32], dv[32], pk[16];
                    tmem_ld32(t_s + 32u * b, sv);
                    tmem_ld32(t_dp + 32u * b, dv);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float ds[2];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int j = ks + 32 * b + e + q;
                            float pr = 0.f;
                            if (valid && j >= lo && j <= i)
                                pr = bt_ex2(fmaf(__uint_as_float(sv[e + q]), C, -lse2));
                            ds[q] = pr * (__uint_as_float(dv[e + q]) - D);
                        }
                        pk[e >> 1] = bt_pack_f16(ds[0], ds[1]);
                    }
                    tmem_st16(t_s + 16u * b + 32u * half, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(T_DS_READY));
            }
            if (!alive) break;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(T_ACC_FULL), aph, abort_flag, status))) break;
            aph ^= 1;
            tc_fence_after();
            float* dst = p.dq + ((size_t)i * kHQ + h) * kHD;
#pragma unroll 1
            for (int b = 2 * half; b < 2 * half + 2; ++b) {
                uint32_t v[32];
                tmem_ld32(t_dq + 32u * b, v);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(dst + 32 * b + e) =
                            make_float4(__uint_as_float(v[e]) * dqs, __uint_as_float(v[e + 1]) * dqs,
                                        __uint_as_float(v[e + 2]) * dqs, __uint_as_float(v[e + 3]) * dqs);
                }
            }
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ============================================================================ dk, dv
__global__ void __launch_bounds__(kBtThreads, 1)
bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_v,
                  const BwdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kDkOffBar;
    auto bar = [&](uint32_t i) { return bar0 + 8u * i; };
    BtMisc* misc = reinterpret_cast<BtMisc*>(smem + kDkOffBar + kBtOffMisc);
    float* colv = reinterpret_cast<float*>(smem + kDkOffCol);      // [stage][lse2 128 | D 128]
    volatile int* abort_flag = &misc->abort_flag;
    int* status = p.status;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tiles = (p.T + 127) / 128;
    const int n_units = n_tiles * kHKV * p.np;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(T_SCHED_FULL + s), 1);
            mbar_init(bar(T_SCHED_EMPTY + s), 1 + 8);
            mbar_init(bar(T_A_FULL + s), 1);
            mbar_init(bar(T_A_EMPTY + s), 1);
        }
        mbar_init(bar(T_B_FULL), 1);
        mbar_init(bar(T_B_EMPTY), 1);
        mbar_init(bar(T_S_FULL), 1);
        mbar_init(bar(T_DS_READY), 256);
        mbar_init(bar(T_ACC_FULL), 1);
        mbar_init(bar(T_DRAIN), 1);
        mbar_init(bar(T_GO), 1);
        mbar_init(bar(T_FIX), 256);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&misc->tmem_base), 512);
        tmem_relinquish();
    }
    if (warp == 2) bt_setup_scales(p, misc, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ scheduler + producer (whole warp)
        uint32_t sslot = 0, sph = 0, kvph = 0, st = 0, ph = 0, narm_kv = 0, narm = 0;
        int last_kt = -1, kqb = 0, kqe = 0;           // query range of the last key tile seen
        bool ok = true;
        for (;;) {
            // next non-empty unit: piece pc of key tile kt for KV head g,
            // u = (kt * np + pc) * 4 + g, query tiles [pc qp, (pc+1) qp) of the
            // tile's range
            int u = -1, qb = 0, nqt = 0, pc = 0;
            if (lane == 0) {
                for (;;) {
                    u = atomicAdd(p.counter, 1);
                    if (u >= n_units) { u = -1; break; }
                    const int kt = u / (kHKV * p.np);
                    pc = (u / kHKV) % p.np;
                    if (kt != last_kt) {
                        k_tile_queries(p, kt * 128, &kqb, &kqe);
                        last_kt = kt;
                    }
                    const int ntot = (kqe - kqb + kTokPerTile - 1) / kTokPerTile;
                    if (pc * p.qp < ntot) {
                        qb = kqb + kTokPerTile * p.qp * pc;
                        nqt = min(p.qp, ntot - pc * p.qp);
                        break;
                    }
                }
            }
            u = __shfl_sync(0xffffffffu, u, 0);
            qb = __shfl_sync(0xffffffffu, qb, 0);
            nqt = __shfl_sync(0xffffffffu, nqt, 0);
            pc = __shfl_sync(0xffffffffu, pc, 0);
            if (!__all_sync(0xffffffffu, mbar_wait(bar(T_SCHED_EMPTY + sslot), sph ^ 1, abort_flag, status)))
                break;
            if (lane == 0) {
                misc->sched[sslot][0] = u;
                misc->sched[sslot][1] = qb;
                misc->sched[sslot][2] = nqt;
                misc->sched[sslot][3] = pc;
                mbar_arrive(bar(T_SCHED_FULL + sslot));
            }
            __syncwarp();
            sslot ^= 1; if (sslot == 0) sph ^= 1;
            if (u < 0) break;
            const int g = u % kHKV, j0 = (u / (kHKV * p.np)) * 128;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(T_B_EMPTY), kvph ^ 1, abort_flag, status));
            if (!ok) break;
            if (lane == 0) {
                mbar_expect_tx(bar(T_B_FULL), 2 * kBtTile);
                tma_load_3d(sbase + kDkOffK, &tm_kh, bar(T_B_FULL), 0, g, j0);
                tma_load_3d(sbase + kDkOffK + kBtHalf, &tm_kh, bar(T_B_FULL), 64, g, j0);
                tma_load_3d(sbase + kDkOffV, &tm_v, bar(T_B_FULL), 0, g, j0);
                tma_load_3d(sbase + kDkOffV + kBtHalf, &tm_v, bar(T_B_FULL), 64, g, j0);
            }
            ++narm_kv;
            kvph ^= 1;
            for (int t = 0; t < nqt && ok; ++t) {
                const int i0 = qb + kTokPerTile * t;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(T_A_EMPTY + st), ph ^ 1, abort_flag, status));
                if (!ok) break;
                // lse2 and D of the tile's 128 columns (token i0 + n/8, head 8g + n%8)
                float* cv = colv + st * 256;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int n = lane + 32 * k;
                    const int i = i0 + (n >> 3), h = kGroup * g + (n & 7);
                    float l2 = 0.f, d = 0.f;
                    if (i < p.T) {
                        l2 = p.lse[(size_t)h * p.T + i] * 1.4426950408889634f;
                        d = p.delta[(size_t)i * kHQ + h];
                    }
                    cv[n] = l2;
                    cv[128 + n] = d;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_expect_tx(bar(T_A_FULL + st), 2 * kBtTile);
                    const uint32_t dq_ = sbase + kDkOffQ + st * kBtTile, ddo = sbase + kDkOffDo + st * kBtTile;
                    tma_load_3d(dq_, &tm_qh, bar(T_A_FULL + st), 0, kGroup * g, i0);
                    tma_load_3d(dq_ + kBtHalf, &tm_qh, bar(T_A_FULL + st), 64, kGroup * g, i0);
                    tma_load_3d(ddo, &tm_do, bar(T_A_FULL + st), 0, kGroup * g, i0);
                    tma_load_3d(ddo + kBtHalf, &tm_do, bar(T_A_FULL + st), 64, kGroup * g, i0);
                }
                ++narm;
                st ^= 1; if (st == 0) ph ^= 1;
            }
            if (!ok) break;
        }
        if (lane == 0) {
            volatile int never = 0;
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            if (narm_kv) mbar_wait(bar(T_B_FULL), (narm_kv - 1) & 1, &never, nullptr, lim);
            for (uint32_t s = 0; s < 2; ++s) {
                const uint32_t n = (narm + 1 - s) / 2;
                if (n) mbar_wait(bar(T_A_FULL + s), (n - 1) & 1, &never, nullptr, lim);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_f16(0, 0, 0, 128);     // Kh x Qh^T (FP16)
            const uint32_t id_dp = idesc_f16(1, 1, 0, 128);    // V x dO^T (BF16)
            const uint32_t id_dv = idesc_f16(1, 1, 1, 128);    // P^T (TMEM, BF16) x dO, MN-major B
            const uint32_t id_dk = idesc_f16(0, 0, 1, 128);    // dS^T (TMEM, FP16) x Qh, MN-major B
            const uint64_t dk0 = smem_desc_sw128(sbase + kDkOffK, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + kDkOffV, 16, 1024);
            const uint64_t dq0 = smem_desc_sw128(sbase + kDkOffQ, 16, 1024);
            const uint64_t ddo = smem_desc_sw128(sbase + kDkOffDo, 16, 1024);
            const uint64_t dqm = smem_desc_sw128(sbase + kDkOffQ, kBtHalf, 1024);
            const uint64_t ddom = smem_desc_sw128(sbase + kDkOffDo, kBtHalf, 1024);
            constexpr uint32_t kStep = kBtTile >> 4;
            uint32_t sslot = 0, sph = 0, kvph = 0, st = 0, ph = 0, dsph = 0;
            bool ok = true;
            for (; ok;) {
                if (!mbar_wait(bar(T_SCHED_FULL + sslot), sph, abort_flag, status)) break;
                const int u = misc->sched[sslot][0];
                const int nqt = misc->sched[sslot][2];
                mbar_arrive(bar(T_SCHED_EMPTY + sslot));
                sslot ^= 1; if (sslot == 0) sph ^= 1;
                if (u < 0) break;
                if (nqt == 0) continue;
                if (!mbar_wait(bar(T_B_FULL), kvph, abort_flag, status)) break;
                kvph ^= 1;
                for (int t = 0; t < nqt; ++t) {
                    ok = mbar_wait(bar(T_A_FULL + st), ph, abort_flag, status);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * (kBtHalf >> 4) + (kk & 3) * 2;
                        mma_ss(tmem, dk0 + off, dq0 + st * kStep + off, id_s, kk > 0);
                    }
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * (kBtHalf >> 4) + (kk & 3) * 2;
                        mma_ss(tmem + 128, dv0 + off, ddo + st * kStep + off, id_dp, kk > 0);
                    }
                    mma_commit(bar(T_S_FULL));
                    ok = mbar_wait(bar(T_DS_READY), dsph, abort_flag, status);
                    if (!ok) break;
                    dsph ^= 1;
                    tc_fence_after();
                    // dV += P^T dO, dK += dS^T Qh (K = 128 query rows, 8 steps
                    // of 16; P^T and dS^T in TMEM: query columns 0..63 packed
                    // into columns 0..31 of their region, 64..127 into 64..95)
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + 256, tmem + 8 * kk + (kk >= 4 ? 32u : 0u), ddom + st * kStep + kk * (2048 >> 4),
                               id_dv, (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + 384, tmem + 128 + 8 * kk + (kk >= 4 ? 32u : 0u),
                               dqm + st * kStep + kk * (2048 >> 4), id_dk, (t > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(T_A_EMPTY + st));
                    st ^= 1; if (st == 0) ph ^= 1;
                }
                if (!ok) break;
                mma_commit(bar(T_B_EMPTY));
                mma_commit(bar(T_ACC_FULL));
            }
            mma_commit(bar(T_DRAIN));
            volatile int never = 0;
            mbar_wait(bar(T_DRAIN), 0, &never, nullptr, 100ull * 1000ull * 1000ull);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ key rows: P^T, dS^T, then dk~, dv
        // Two warpgroups: warps 4-7 take the query columns 0..63 of every
        // key row, warps 8-11 the columns 64..127 (each writes its P^T and
        // dS^T inside its own columns), and each stores half of dk~ and dv.
        const int half = (warp - 4) >> 2;
        const int r = (tid - 128) & 127;                // TMEM lane = key row
        const uint32_t lb = (uint32_t)(warp & 3) * 32u;
        const uint32_t t_s = tmem + (lb << 16), t_dp = t_s + 128, t_dv = t_s + 256, t_dk = t_s + 384;
        const float C = misc->logit_scale, dks = misc->dk_scale;
        uint32_t sslot = 0, sph = 0, s_ph = 0, aph = 0, st = 0, ph = 0, gph = 0, fph = 0;
        for (;;) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(T_SCHED_FULL + sslot), sph, abort_flag, status))) break;
            const int u = misc->sched[sslot][0];
            const int qb = misc->sched[sslot][1], nqt = misc->sched[sslot][2];
            const int pc = misc->sched[sslot][3];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(T_SCHED_EMPTY + sslot));
            sslot ^= 1; if (sslot == 0) sph ^= 1;
            if (u < 0) break;
            if (nqt == 0) continue;
            const int g = u % kHKV, kt = u / (kHKV * p.np), j = kt * 128 + r;
            const bool valid = j < p.T && p.seg_lo[j] >= 0;
            int hi = 0;
            if (valid) hi = p.window > 0 ? min(p.seg_hi[j], j + p.window) : p.seg_hi[j];
            bool alive = true;
            for (int t = 0; t < nqt; ++t) {
                // S^T and dP^T of this query tile; its lse2 / D landed with it
                if (!__all_sync(0xffffffffu, mbar_wait(bar(T_S_FULL), s_ph, abort_flag, status))) {
                    alive = false;
                    break;
                }
                s_ph ^= 1;
                // the producer stored this stage's lse2 / D before arming its
                // barrier: acquire that phase too (it has completed already)
                if (!__all_sync(0xffffffffu, mbar_wait(bar(T_A_FULL + st), ph, abort_flag, status))) {
                    alive = false;
                    break;
                }
                tc_fence_after();
                const float* cv = colv + st * 256;
                const int i0 = qb + kTokPerTile * t;
#pragma unroll 1
                for (int b = 2 * half; b < 2 * half + 2; ++b) {
                    uint32_t sv[32], dv[32], pp[16], pd[16];
                    tmem_ld32(t_s + 32u * b, sv);
                    tmem_ld32(t_dp + 32u * b, dv);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        // lse2 and D of columns 32b + e .. +3 (one broadcast load each)
                        const float4 l4 = *reinterpret_cast<const float4*>(cv + 32 * b + e);
                        const float4 d4 = *reinterpret_cast<const float4*>(cv + 128 + 32 * b + e);
                        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
                        float pr[4], ds[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int n = 32 * b + e + q;            // column: token i0 + n/8, head n%8
                            const int i = i0 + (n >> 3);
                            float x = 0.f;
                            if (valid && i >= j && i < hi)
                                x = bt_ex2(fmaf(__uint_as_float(sv[e + q]), C, -lv[q]));
                            pr[q] = x;
                            ds[q] = x * (__uint_as_float(dv[e + q]) - dd[q]);
                        }
                        pp[e >> 1] = bt_pack_bf16(pr[0], pr[1]);
                        pp[(e >> 1) + 1] = bt_pack_bf16(pr[2], pr[3]);
                        pd[e >> 1] = bt_pack_f16(ds[0], ds[1]);
                        pd[(e >> 1) + 1] = bt_pack_f16(ds[2], ds[3]);
                    }
                    tmem_st16(t_s + 16u * b + 32u * half, pp);
                    tmem_st16(t_dp + 16u * b + 32u * half, pd);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(T_DS_READY));
                st ^= 1; if (st == 0) ph ^= 1;
            }
            if (!alive) break;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(T_ACC_FULL), aph, abort_flag, status))) break;
            aph ^= 1;
            // Pieces of one key tile and head are summed in piece order, so
            // the result does not depend on which CTA ran which piece: piece
            // pc > 0 waits until piece pc - 1 has stored, then adds to it.
            // Every piece was dispensed after its predecessor (lower unit
            // index) to a CTA that is running, so the wait ends.
            int* flag = p.flags + kt * kHKV + g;
            if (pc > 0) {
                if (tid == 128) {
                    misc->fix_ok = flag_wait_geq(flag, pc, abort_flag, status) ? 1 : 0;
                    mbar_arrive(bar(T_GO));
                }
                __syncwarp();
                if (!__all_sync(0xffffffffu, mbar_wait(bar(T_GO), gph, abort_flag, status))) break;
                gph ^= 1;
                if (!misc->fix_ok) break;
            }
            tc_fence_after();
            float* dkd = p.dk + ((size_t)j * kHKV + g) * kHD;
            float* dvd = p.dv + ((size_t)j * kHKV + g) * kHD;
#pragma unroll 1
            for (int b = 2 * half; b < 2 * half + 2; ++b) {
                uint32_t a[32], c[32];
                tmem_ld32(t_dk + 32u * b, a);
                tmem_ld32(t_dv + 32u * b, c);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        float4 k4 = make_float4(__uint_as_float(a[e]) * dks, __uint_as_float(a[e + 1]) * dks,
                                                __uint_as_float(a[e + 2]) * dks, __uint_as_float(a[e + 3]) * dks);
                        float4 v4 = make_float4(__uint_as_float(c[e]), __uint_as_float(c[e + 1]),
                                                __uint_as_float(c[e + 2]), __uint_as_float(c[e + 3]));
                        if (pc > 0) {
                            // the earlier pieces' sum, from L2 (written by another SM)
                            const float4 k0 = __ldcg(reinterpret_cast<const float4*>(dkd + 32 * b + e));
                            const float4 v0 = __ldcg(reinterpret_cast<const float4*>(dvd + 32 * b + e));
                            k4 = make_float4(k0.x + k4.x, k0.y + k4.y, k0.z + k4.z, k0.w + k4.w);
                            v4 = make_float4(v0.x + v4.x, v0.y + v4.y, v0.z + v4.z, v0.w + v4.w);
                        }
                        __stcg(reinterpret_cast<float4*>(dkd + 32 * b + e), k4);
                        __stcg(reinterpret_cast<float4*>(dvd + 32 * b + e), v4);
                    }
                }
            }
            tc_fence_before();
            // this piece's rows are stored: publish pc + 1 for the next piece
            mbar_arrive(bar(T_FIX));
            if (tid == 128 && mbar_wait(bar(T_FIX), fph, abort_flag, status)) flag_release(flag, pc + 1);
            __syncwarp();
            fph ^= 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ============================================================================ host
namespace {

// 3-D map over a [T, heads, 128] tensor of 16-bit elements: dims (128, heads,
// T), box (64, box_heads, box_tokens), 128-byte swizzle, zero fill outside.
flint_status_t bt_map(EncodeTiledFn enc, CUtensorMap* m, CUtensorMapDataType dt, const void* base, int heads,
                      int T, int box_heads, int box_tokens) {
    cuuint64_t dims[3] = {(cuuint64_t)kHD, (cuuint64_t)heads, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)kHD * 2, (cuuint64_t)heads * kHD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return FLINT_OK;
}

bool g_bt_attr[64] = {false};

}  // namespace

// Pieces of a key tile's query range for the dk/dv kernel: on short
// sequences the key tiles (4 per 128 tokens) are too few to balance over the
// SMs, and on a causal sequence the first tile sees every query while the
// last sees 128, so each tile's range is cut into up to `np` pieces of `qp`
// query tiles, about 4 units per SM.  Long sequences keep one piece per tile.
void bwd_pieces(int T, int window, int sms, int* qp, int* np) {
    const int n_kt = (T + 127) / 128;
    const int units = n_kt * kHKV;
    // query tiles a key tile can see, at most (its range starts at its
    // first valid key, not on a tile boundary)
    int nqt_max = (T + kTokPerTile - 1) / kTokPerTile + 1;
    if (window > 0) nqt_max = min(nqt_max, (128 + window + kTokPerTile - 2) / kTokPerTile + 1);
    const int target = (4 * sms + units - 1) / (units > 0 ? units : 1);
    if (target <= 1) {
        *qp = nqt_max;
        *np = 1;
        return;
    }
    int q = (nqt_max + target - 1) / target;
    if (q < 8) q = 8;
    *qp = q;
    *np = (nqt_max + q - 1) / q;
}

// Enqueues the two tensor-core kernels.  qh [T,32,128] and kh [T,4,128] are
// the FP16 scaled operands (2^eq q~, 2^ek k~); counters: two zeroed ints;
// flags: ceil(T/128) x 4 zeroed ints.
flint_status_t launch_bwd_tc(const void* qh, const void* kh, const void* v, const void* dout,
                             const float* q_norm_w, const float* k_norm_w, const float* lse,
                             const float* delta, const int* seg_lo, const int* seg_hi, float* dq, float* dk,
                             float* dv, int* status, int* counters, int* flags, int T, int window, int sms,
                             cudaStream_t s) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return fail(FLINT_ERR_UNSUPPORTED, "device index %d", dev);
    if (!g_bt_attr[dev]) {
        cudaError_t e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kBtSmemDq);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kBtSmemDk);
        if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        g_bt_attr[dev] = true;
    }
    EncodeTiledFn enc = nullptr;
    flint_status_t st = get_encoder(&enc);
    if (st != FLINT_OK) return st;
    CUtensorMap tq, tdo, tk, tv;
    st = bt_map(enc, &tq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, qh, kHQ, T, kGroup, kTokPerTile);
    if (st == FLINT_OK) st = bt_map(enc, &tdo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dout, kHQ, T, kGroup, kTokPerTile);
    if (st == FLINT_OK) st = bt_map(enc, &tk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, kh, kHKV, T, 1, 128);
    if (st == FLINT_OK) st = bt_map(enc, &tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, kHKV, T, 1, 128);
    if (st != FLINT_OK) return st;
    BwdTcParams p;
    p.q_norm_w = q_norm_w;
    p.k_norm_w = k_norm_w;
    p.lse = lse;
    p.delta = delta;
    p.seg_lo = seg_lo;
    p.seg_hi = seg_hi;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.status = status;
    p.flags = flags;
    p.T = T;
    p.window = window;
    bwd_pieces(T, window, sms, &p.qp, &p.np);
    const int units_q = ((T + kTokPerTile - 1) / kTokPerTile) * kHKV;
    const int units_k = ((T + 127) / 128) * kHKV * p.np;
    p.counter = counters;
    bwd_dq_tc_kernel<<<units_q < sms ? units_q : sms, kBtThreads, kBtSmemDq, s>>>(tq, tdo, tk, tv, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "backward dq launch: %s", cudaGetErrorString(e));
    p.counter = counters + 1;
    bwd_dkv_tc_kernel<<<units_k < sms ? units_k : sms, kBtThreads, kBtSmemDk, s>>>(tq, tdo, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "backward dk/dv launch: %s", cudaGetErrorString(e));
    return FLINT_OK;
}

}  // namespace flint
