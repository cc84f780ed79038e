// Tensor-core decode step (sm_100a: TMA, tcgen05, TMEM) for the common case
// of a logit bound <= 48 (decode_logit_bound).  Same operation as the
// CUDA-core split kernel in flint_decode.cu (FlintAttention.forward on the
// NeMo AutoModel "flint.layers" API page, applied to one new token per
// sequence against its key/value cache; the sink as a zero-value softmax
// column, HF discussion #26 on RecursiveSI/flint), reorganised so that the
// step streams the cache at HBM speed:
//
// * A persistent CTA per SM takes work items (sequence b, KV head g, split):
//   its own index first, then the rest from a counter, each published to the
//   CTA's warps with its position.  A split is a run of 128-slot tiles of the
//   cache; tiles with no slot in the token's window are skipped.  Slot s
//   holds position pos - ((pos - s) mod cap), which is in the window when
//   (pos - s) mod cap < n = pos - lo + 1.
// * Warp 0 streams the K and V tiles by TMA (three 64 KiB stages of K and V,
//   128-byte swizzle, the same layout as the attention kernel's tiles) ahead
//   of the MMAs, across items, and prefetches the next item's q, k, v rows
//   into L2 (the first item's at kernel entry, before the first tiles).
// * Warp 1 issues, per tile, S^T = K Q^T (M = 128 slots, N = 16: the 8
//   query heads as BF16 high parts and as the BF16 rounding of the
//   remainders, so hi + lo carries q~ to about 2^-17) and, once the slot
//   rows have written P, O^T += V^T P^T (M = 128 channels with V read
//   M-major, N = 16 with the 8 heads' P in BF16, K = 128 slots), both
//   accumulated in FP32 in TMEM.
// * Warps 4-7 take one slot row each: the score of each head is the sum of
//   its hi and lo columns; with the running max started at the bound B
//   (every term 2^(s - B) <= 1 and normal) no row max and no rescale are
//   needed, so a split's partial is (m = B, l = sum of terms, O).  An
//   item's end (O^T out of TMEM, the output or the partial) waits until the
//   next item's first tile is with the MMA, so the tiles of consecutive
//   items follow each other without a wait for the last PV.
// * Warps 2-3 prepare each item one ahead of the slot rows, into buffers of
//   the item's parity: q~ (norm, RoPE) of 8 heads as the hi/lo rows of Q^T,
//   the new token's k~ (FP32) and its scores against the 8 heads, and the
//   append of k~ (BF16) and v to slot pos mod cap.  The slot row of that tile
//   takes the FP32 score and the new value (written into the V tile before
//   the PV MMA), whatever the cache held when the tile was loaded.
// * A split that is the whole window writes the output and LSE itself;
//   otherwise the last split of (b, g) to finish folds them (decode_fold).
// Every wait is bounded (FLINT_ERR_TIMEOUT in the status word, abort, drain).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "../../include/flint_attn.h"
#include "flint_common.cuh"
#include "flint_decode.cuh"
#include "flint_host.cuh"
#include "sm100.cuh"

namespace flint {

constexpr int kDtThreads = 256;
constexpr uint32_t kDtHalf = kDtSlots * 128;          // one 64-channel half of a tile: 16 KiB
constexpr uint32_t kDtTile = 2 * kDtHalf;             // K or V tile: 32 KiB
constexpr uint32_t kDtStage = 2 * kDtTile;            // K + V
constexpr uint32_t kDtStages = 3;
constexpr uint32_t kDtB16Half = 16 * 128;              // one 64-column half of a 16-row B operand
constexpr uint32_t kDtOffP = kDtStages * kDtStage;     // 2 P^T buffers (B operand, 16 rows x 128 slots)
constexpr uint32_t kDtOffQt = kDtOffP + 2 * 2 * kDtB16Half;   // Q^T (B operand, 16 rows x 128 channels)
constexpr uint32_t kDtQtHalf = kDtB16Half;
constexpr uint32_t kDtQtBytes = 2 * kDtQtHalf;                // one Q^T buffer (two per item parity)
constexpr uint32_t kDtOffInv = kDtOffQt + 2 * kDtQtBytes;     // 64 RoPE inverse frequencies (double)
constexpr uint32_t kDtOffMisc = kDtOffInv + 64 * 8;
constexpr uint32_t kDtOffBar = kDtOffMisc + 512;
constexpr uint32_t kDtNumBars = 32;
constexpr uint32_t kDtSmem = kDtOffBar + 8 * kDtNumBars + 1024;
static_assert(kDtSmem <= 232448, "shared memory per block");

enum : uint32_t {
    D_FULL = 0, D_EMPTY = 3,            // stages
    D_SCHED_FULL = 6, D_SCHED_EMPTY = 8,
    D_S_FULL = 10, D_P_READY = 12, D_P_FREE = 14,
    // per item parity: Q^T and the new token's scores written (query warps);
    // the item's tiles done (slot rows); O^T complete (MMA); O^T read (slot rows)
    D_ITEM_READY = 16, D_ITEM_DONE = 18, D_O_FULL = 20, D_O_FREE = 22,
    D_L_READY = 24, D_DRAIN = 25,
    D_FOLD_A = 26, D_FOLD_B = 27        // slot rows: partial written; last-split decision
};

struct DtMisc {
    int sched[2];
    int sched_pos[2];                   // the scheduled item's position (cache_len of its sequence)
    uint32_t tmem_base;
    int abort_flag;
    float bound;                        // B, log2 units
    float s_new[2][8];                  // per item parity: the new token's scores, per head (unscaled)
    float red_l[2][4][8];               // per item parity and slot-row warp: its part of l, per head
    int last;                           // this split is the last of its (b, g) to finish
    int first_pos;                      // the first item's position (read early, for its cache line)
    float sinks[kHQ];                   // the learned sinks
};
static_assert(sizeof(DtMisc) <= 512, "misc block");

// Work item -> sequence, KV head, split, and the split's tile range.
struct DtItem {
    int b, g, t0, t1;                   // tiles [t0, t1)
    int pos, lo, n;                     // new token's position, window start, window length
    bool bad;                           // ill-formed position or window
};

__device__ __forceinline__ DtItem dt_item(const DecodeParams& p, int i, int pos) {
    DtItem it;
    const int ns = p.nsplit_tc;
    it.b = i / (kHKV * ns);
    it.g = (i / ns) % kHKV;
    const int sp = i % ns;
    const int nt = decode_tc_tiles(p.cap), per = decode_tc_tiles_per_split(p.cap);
    it.t0 = sp * per;
    it.t1 = min(nt, it.t0 + per);
    it.pos = pos;
    it.lo = p.window > 0 ? max(0, it.pos - p.window + 1) : 0;
    it.n = it.pos - it.lo + 1;
    it.bad = it.pos < 0 || it.pos >= FLINT_MAX_TOKENS || it.n > p.cap;
    return it;
}

// Whether tile t holds a slot of the window: the cyclic slot interval
// [lo mod cap, lo mod cap + n) meets [128 t, min(128 t + 128, cap)).
__device__ __forceinline__ bool dt_tile_live(const DecodeParams& p, const DtItem& it, int t) {
    if (it.bad) return false;
    if (it.n >= p.cap) return true;
    const int a = it.lo % p.cap, e = a + it.n;
    const int s0 = t * kDtSlots, s1 = min(s0 + kDtSlots, p.cap);
    return (max(a, s0) < min(e, s1)) || (max(a, s0 + p.cap) < min(e, s1 + p.cap));
}

__device__ __forceinline__ float dt_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Byte offset of element (row, col) of a K-major operand tile stored as two
// 64-column halves of 128-byte rows, 128-byte swizzle (the TMA layout).
__device__ __forceinline__ uint32_t dt_sw_off(int row, int col, uint32_t half_bytes) {
    const int h = col >> 6, cc = col & 63;
    return (uint32_t)h * half_bytes + (uint32_t)row * 128u + ((uint32_t)(((cc >> 3) ^ (row & 7))) << 4) +
           (uint32_t)(cc & 7) * 2u;
}

__global__ void __launch_bounds__(kDtThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                 const DecodeParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kDtOffBar;
    auto bar = [&](uint32_t i) { return bar0 + 8u * i; };
    DtMisc* misc = reinterpret_cast<DtMisc*>(smem + kDtOffMisc);
    volatile int* abort_flag = &misc->abort_flag;
    int* status = p.status;
    int* counter = p.status + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_items = p.B * kHKV * p.nsplit_tc;
    // The CUDA-core split kernel behind this one may be scheduled now: it
    // reads the weights and returns, or waits for this grid.
    griddep_launch_dependents();
    // Each CTA's first item is its own index (later ones come from the
    // counter), so its rows can be on their way to L2 before every CTA's
    // first cache tiles fill the memory queues: the query warps' loads of
    // them would otherwise wait behind those.
    if (warp == 2 && lane == 0 && (int)blockIdx.x < n_items) {
        const int fb = (int)blockIdx.x / (kHKV * p.nsplit_tc), fg = ((int)blockIdx.x / p.nsplit_tc) % kHKV;
        bulk_prefetch_l2(p.q + ((size_t)fb * kHQ + kGroup * fg) * kHD, kGroup * kHD * 2);
        bulk_prefetch_l2(p.k + ((size_t)fb * kHKV + fg) * kHD, kHD * 2);
        bulk_prefetch_l2(p.v + ((size_t)fb * kHKV + fg) * kHD, kHD * 2);
        misc->first_pos = p.cache_len[fb];    // its line, too
    }

    // this kernel runs only under a logit bound <= 48; otherwise the
    // CUDA-core split kernel does the step (every CTA decides the same way)
    if (warp == 0) {
        const float bnd = decode_logit_bound(p.q_norm_w, p.k_norm_w);
        if (lane == 0) misc->bound = bnd;
    }
    __syncthreads();
    if (!(misc->bound <= kDecodeBoundMax)) {
        // the split kernel waits for this grid only: this grid's end must
        // come after the header reset
        griddep_wait();
        return;
    }

    if (tid == 0) {
        for (uint32_t s = 0; s < kDtStages; ++s) {
            mbar_init(bar(D_FULL + s), 1);
            mbar_init(bar(D_EMPTY + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(D_SCHED_FULL + s), 1);
            mbar_init(bar(D_SCHED_EMPTY + s), 1 + 2 + 4);   // MMA, query warps, slot-row warps (lane 0)
            mbar_init(bar(D_S_FULL + s), 1);
            mbar_init(bar(D_P_READY + s), 128);
            mbar_init(bar(D_P_FREE + s), 1);
            mbar_init(bar(D_ITEM_READY + s), 64);
            mbar_init(bar(D_ITEM_DONE + s), 128);
            mbar_init(bar(D_O_FULL + s), 1);
            mbar_init(bar(D_O_FREE + s), 128);
        }
        mbar_init(bar(D_L_READY), 128);
        mbar_init(bar(D_DRAIN), 1);
        mbar_init(bar(D_FOLD_A), 128);
        mbar_init(bar(D_FOLD_B), 128);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_kc);
        tma_prefetch_desc(&tm_vc);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&misc->tmem_base), 128);
        tmem_relinquish();
    }
    double* inv_freq = reinterpret_cast<double*>(smem + kDtOffInv);
    if (warp == 3) misc->sinks[lane] = p.sinks[lane];
    if (warp == 2) {
        const double l2t = log2((double)p.rope_theta);
        inv_freq[lane] = exp2(-(double)lane / 64.0 * l2t);
        inv_freq[lane + 32] = exp2(-(double)(lane + 32) / 64.0 * l2t);
    }
    // P^T rows 8..15 stay zero (only the 8 heads' rows are written)
    for (uint32_t o = (uint32_t)tid * 16u; o < 4 * kDtB16Half; o += kDtThreads * 16u) {
        const uint32_t row = (o % kDtB16Half) / 128u;
        if (row >= 8) *reinterpret_cast<uint4*>(smem + kDtOffP + o) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    // the status word, the work counter and the split-arrival counters are
    // read and written only after the reset kernel before this one completed
    griddep_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const float B = misc->bound;

    if (warp == 0) {
        // ------------------------------------------------ scheduler + TMA producer
        if (lane == 0) {
            uint32_t sslot = 0, sph = 0, st = 0, ph = 0, narm = 0;
            // items are published one ahead of the item being loaded, so the
            // query warps prepare the next item while this one streams
            // with the item, its position: the consumers take it from here
            // instead of each reading cache_len at every item change
            auto publish = [&](int v, int vpos) -> bool {
                if (!mbar_wait(bar(D_SCHED_EMPTY + sslot), sph ^ 1, abort_flag, status)) return false;
                misc->sched[sslot] = v;
                misc->sched_pos[sslot] = vpos;
                mbar_arrive(bar(D_SCHED_FULL + sslot));
                sslot ^= 1; if (sslot == 0) sph ^= 1;
                return true;
            };
            // the first item is the CTA's index; the counter hands out the
            // rest, from gridDim.x on
            int u = (int)blockIdx.x < n_items ? (int)blockIdx.x : -1;
            int upos = u >= 0 ? p.cache_len[u / (kHKV * p.nsplit_tc)] : 0;
            bool pub = publish(u, upos);
            for (; pub;) {
                if (u < 0) break;
                int un = atomicAdd(counter, 1) + (int)gridDim.x;
                if (un >= n_items) un = -1;
                const int unpos = un >= 0 ? p.cache_len[un / (kHKV * p.nsplit_tc)] : 0;
                if (!publish(un, unpos)) break;
                if (un >= 0) {
                    // the next item's q, k and v rows into L2 (its prologue reads them)
                    const int nb = un / (kHKV * p.nsplit_tc), ng = (un / p.nsplit_tc) % kHKV;
                    bulk_prefetch_l2(p.q + ((size_t)nb * kHQ + kGroup * ng) * kHD, kGroup * kHD * 2);
                    bulk_prefetch_l2(p.k + ((size_t)nb * kHKV + ng) * kHD, kHD * 2);
                    bulk_prefetch_l2(p.v + ((size_t)nb * kHKV + ng) * kHD, kHD * 2);
                }
                const DtItem it = dt_item(p, u, upos);
                bool ok = true;
                for (int t = it.t0; t < it.t1 && ok; ++t) {
                    if (!dt_tile_live(p, it, t)) continue;
                    ok = mbar_wait(bar(D_EMPTY + st), ph ^ 1, abort_flag, status);
                    if (!ok) break;
                    const uint32_t dst = sbase + st * kDtStage;
                    mbar_expect_tx(bar(D_FULL + st), kDtStage);
                    const int bg = it.b * kHKV + it.g;
                    tma_load_3d(dst, &tm_kc, bar(D_FULL + st), 0, t * kDtSlots, bg);
                    tma_load_3d(dst + kDtHalf, &tm_kc, bar(D_FULL + st), 64, t * kDtSlots, bg);
                    tma_load_3d(dst + kDtTile, &tm_vc, bar(D_FULL + st), 0, t * kDtSlots, bg);
                    tma_load_3d(dst + kDtTile + kDtHalf, &tm_vc, bar(D_FULL + st), 64, t * kDtSlots, bg);
                    ++narm;
                    if (++st == kDtStages) { st = 0; ph ^= 1; }
                }
                if (!ok) break;
                u = un;
                upos = unpos;
            }
            // drain: every armed load has landed before shared memory is released
            volatile int never = 0;
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            for (uint32_t s2 = 0; s2 < kDtStages; ++s2) {
                // stage s2 received loads number s2, s2 + 3, ...
                const uint32_t nl = (narm + kDtStages - 1 - s2) / kDtStages;
                if (nl) mbar_wait(bar(D_FULL + s2), (nl - 1) & 1, &never, nullptr, lim);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_f16(1, 1, 0, 16);      // K x Q^T: BF16, N = 16
            const uint32_t id_o = idesc_f16_amn(1, 1, 16);     // V^T x P^T: BF16, V read M-major, N = 16
            uint32_t sslot = 0, sph = 0, st = 0, ph = 0, tt = 0, k_item = 0;
            uint32_t prph[2] = {0u, 0u}, irph[2] = {0u, 0u}, ofph[2] = {0u, 0u};
            bool ok = true;
            uint32_t ob = 0;                     // O^T buffer of the current item
            // O^T += V^T(stage pst) P^T(tile ptt); its P is ready
            auto issue_pv = [&](uint32_t pst, uint32_t ptt, bool acc) {
                const uint32_t pb = ptt & 1u;
                const uint64_t dv = smem_desc_sw128(sbase + pst * kDtStage + kDtTile, kDtHalf, 1024);
                const uint64_t dp = smem_desc_sw128(sbase + kDtOffP + pb * 2 * kDtB16Half, 16, 1024);
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk) {
                    const uint32_t off_b = (kk >> 2) * (kDtB16Half >> 4) + (kk & 3) * 2;
                    mma_ss(tmem + 64 + 32 * ob, dv + kk * (2048 >> 4), dp + off_b, id_o, (acc || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(D_EMPTY + pst));
                mma_commit(bar(D_P_FREE + pb));
            };
            for (; ok;) {
                if (!mbar_wait(bar(D_SCHED_FULL + sslot), sph, abort_flag, status)) break;
                const int u = misc->sched[sslot], upos = misc->sched_pos[sslot];
                mbar_arrive(bar(D_SCHED_EMPTY + sslot));
                sslot ^= 1; if (sslot == 0) sph ^= 1;
                if (u < 0) break;
                const DtItem it = dt_item(p, u, upos);
                int nl = 0;
                for (int t = it.t0; t < it.t1; ++t) nl += dt_tile_live(p, it, t) ? 1 : 0;
                if (nl == 0) continue;
                // buffers of this item's parity: Q^T written; the O^T of two
                // items back read out
                ob = k_item & 1u;
                if (!mbar_wait(bar(D_ITEM_READY + ob), irph[ob], abort_flag, status)) break;
                irph[ob] ^= 1u;
                if (k_item >= 2) {
                    if (!mbar_wait(bar(D_O_FREE + ob), ofph[ob], abort_flag, status)) break;
                    ofph[ob] ^= 1u;
                }
                ++k_item;
                tc_fence_after();
                const uint64_t dq = smem_desc_sw128(sbase + kDtOffQt + ob * kDtQtBytes, 16, 1024);
                // The S^T of tile a runs up to two tiles ahead of the PV of
                // tile b (two S^T buffers); each is issued as soon as its
                // inputs are ready (the tile landed; its slot rows wrote P).
                int a = 0, bp = 0;                        // live tiles whose S^T / PV were issued
                int tS = it.t0;                           // next tile for S^T
                uint32_t stS = st, phS = ph, ttS = tt;    // its stage, phase, running tile number
                uint32_t stP = st, ttP = tt;              // the same for the next PV
                unsigned long long t_last = global_ns();
                while (bp < nl) {
                    bool progress = false;
                    if (a < nl && a < bp + 2) {
                        while (!dt_tile_live(p, it, tS)) ++tS;
                        if (mbar_try(bar(D_FULL + stS), phS)) {
                            tc_fence_after();
                            // S^T = K Q^T into buffer ttS & 1 (K = 128 channels, 8 steps of 16)
                            const uint64_t dk = smem_desc_sw128(sbase + stS * kDtStage, 16, 1024);
#pragma unroll
                            for (uint32_t kk = 0; kk < 8; ++kk) {
                                const uint32_t off_a = (kk >> 2) * (kDtHalf >> 4) + (kk & 3) * 2;
                                const uint32_t off_b = (kk >> 2) * (kDtQtHalf >> 4) + (kk & 3) * 2;
                                mma_ss(tmem + 32u * (ttS & 1u), dk + off_a, dq + off_b, id_s, kk > 0 ? 1u : 0u);
                            }
                            mma_commit(bar(D_S_FULL + (ttS & 1u)));
                            ++a; ++tS; ++ttS;
                            if (++stS == kDtStages) { stS = 0; phS ^= 1; }
                            progress = true;
                        }
                    }
                    if (bp < a && mbar_try(bar(D_P_READY + (ttP & 1u)), prph[ttP & 1u])) {
                        prph[ttP & 1u] ^= 1u;
                        tc_fence_after();
                        issue_pv(stP, ttP, bp > 0);
                        ++bp; ++ttP;
                        if (++stP == kDtStages) stP = 0;
                        progress = true;
                    }
                    if (progress) {
                        t_last = global_ns();
                    } else if (*abort_flag) {
                        ok = false;
                        break;
                    } else if (global_ns() - t_last > kWaitLimitNs) {
                        atomicCAS(status, 0, kStatusTimeout);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                st = stS;
                ph = phS;
                tt = ttS;
                mma_commit(bar(D_O_FULL + ob));
            }
            // drain: every MMA issued so far has completed
            mma_commit(bar(D_DRAIN));
            volatile int never = 0;
            mbar_wait(bar(D_DRAIN), 0, &never, nullptr, 100ull * 1000ull * 1000ull);
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------ query warps
        // One item ahead of the slot rows: q~ of heads 4 qw .. 4 qw + 3 as
        // BF16 hi/lo rows of this item parity's Q^T; the new token's k~
        // (both warps), its scores against those heads, and (warp 2) the
        // append to the cache.  Lane l holds channels l, l+32, l+64, l+96.
        const int qw = warp - 2;
        const bool rope = p.use_rope != 0;
        uint32_t sslot = 0, sph = 0, k_item = 0;
        uint32_t idph[2] = {0u, 0u};
        for (;;) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(D_SCHED_FULL + sslot), sph, abort_flag, status))) break;
            const int u = misc->sched[sslot], upos = misc->sched_pos[sslot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(D_SCHED_EMPTY + sslot));
            sslot ^= 1; if (sslot == 0) sph ^= 1;
            if (u < 0) break;
            const DtItem it = dt_item(p, u, upos);
            int nl = 0;
            for (int t = it.t0; t < it.t1; ++t) nl += dt_tile_live(p, it, t) ? 1 : 0;
            if (nl == 0) continue;
            const uint32_t ib = k_item & 1u;
            // this parity's buffers are free once the item two back is done
            if (k_item >= 2) {
                if (!__all_sync(0xffffffffu, mbar_wait(bar(D_ITEM_DONE + ib), idph[ib], abort_flag, status))) break;
                idph[ib] ^= 1u;
            }
            ++k_item;
            const int s_new = it.pos % p.cap;
            const bool has_new = s_new >= it.t0 * kDtSlots && s_new < it.t1 * kDtSlots;
            uint8_t* qt = smem + kDtOffQt + ib * kDtQtBytes;
            // every row's values in flight before any arithmetic
            float xq[4][4], xk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int hh = 0; hh < 4; ++hh)
                dec_load_row(p.q + ((size_t)it.b * kHQ + kGroup * it.g + 4 * qw + hh) * kHD, lane, xq[hh]);
            if (has_new) dec_load_row(p.k + ((size_t)it.b * kHKV + it.g) * kHD, lane, xk);
            float yk[4] = {0.f, 0.f, 0.f, 0.f};
            if (has_new) dec_norm_rope_vals(xk, p.k_norm_w, p.eps, rope, it.pos, inv_freq, lane, yk);
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                const int h = 4 * qw + hh;
                float yq[4];
                dec_norm_rope_vals(xq[hh], p.q_norm_w, p.eps, rope, it.pos, inv_freq, lane, yq);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = lane + 32 * i;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(yq[i]);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(yq[i] - __bfloat162float(hi));
                    *reinterpret_cast<__nv_bfloat16*>(qt + dt_sw_off(h, c, kDtQtHalf)) = hi;
                    *reinterpret_cast<__nv_bfloat16*>(qt + dt_sw_off(kGroup + h, c, kDtQtHalf)) = lo;
                }
                if (has_new) {
                    float d = yq[0] * yk[0] + yq[1] * yk[1] + yq[2] * yk[2] + yq[3] * yk[3];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                    if (lane == 0) misc->s_new[ib][h] = d;
                }
            }
            if (has_new && qw == 0) {
                const size_t row = (((size_t)it.b * kHKV + it.g) * p.cap + (size_t)s_new) * kHD;
                const __nv_bfloat16* vsrc = p.v + ((size_t)it.b * kHKV + it.g) * kHD;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    p.k_cache[row + lane + 32 * i] = __float2bfloat16_rn(yk[i]);
                    p.v_cache[row + lane + 32 * i] = vsrc[lane + 32 * i];
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(D_ITEM_READY + ib));
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ slot rows
        const int r = tid - 128;                        // TMEM lane = slot row of the tile
        const int wq = warp - 4;                        // this warp's slot of the l partial sums
        const uint32_t lb = (uint32_t)(warp & 3) * 32u;
        const float C = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)
        const bool whole = p.nsplit_tc == 1;            // every split is the whole window
        uint32_t sslot = 0, sph = 0, lph = 0, tt = 0, sst = 0, fph = 0, k_item = 0;
        uint32_t sfph[2] = {0u, 0u}, pfph[2] = {0u, 0u}, irph[2] = {0u, 0u}, oph[2] = {0u, 0u};
        auto part_of = [&](int u, const DtItem& it) -> float* {
            return p.part + (((size_t)it.b * kHKV + it.g) * p.nsplit_tc + (u % p.nsplit_tc)) * kPartFloats;
        };
        // this split's partial is written: the last split of (b, g) to
        // finish folds them all into the output (bounded waits)
        auto finish = [&](int b, int g) -> bool {
            __threadfence();
            mbar_arrive(bar(D_FOLD_A));
            if (!__all_sync(0xffffffffu, mbar_wait(bar(D_FOLD_A), fph, abort_flag, status))) return false;
            if (tid == 128) misc->last = atomicAdd(p.arrive + b * kHKV + g, 1) == p.nsplit_tc - 1;
            mbar_arrive(bar(D_FOLD_B));
            if (!__all_sync(0xffffffffu, mbar_wait(bar(D_FOLD_B), fph, abort_flag, status))) return false;
            fph ^= 1;
            if (misc->last) {
                __threadfence();
                decode_fold(p, b, g, p.nsplit_tc, r);
            }
            return true;
        };
        // The end of an item whose tiles are done and whose l sits in
        // red_l[pib]: O^T out of TMEM once the item's last PV completed, then
        // the output (a split that is the whole window) or the partial and
        // the fold.  It runs once the next item's first tile is with the
        // MMA, by when those PV MMAs have long completed: the slot rows do
        // not wait for them between items.
        bool pending = false;
        DtItem pit = {};
        int pu = 0;
        uint32_t pib = 0;
        auto end_item = [&]() -> bool {
            pending = false;
            float* part = part_of(pu, pit);
            if (!whole && warp == 4 && lane < kGroup) {
                part[lane] = B;
                part[kGroup + lane] = misc->red_l[pib][0][lane] + misc->red_l[pib][1][lane] +
                                      misc->red_l[pib][2][lane] + misc->red_l[pib][3][lane];
            }
            // O^T: TMEM lane = channel r, columns 0..7 = heads
            if (!__all_sync(0xffffffffu, mbar_wait(bar(D_O_FULL + pib), oph[pib], abort_flag, status))) return false;
            oph[pib] ^= 1u;
            tc_fence_after();
            uint32_t o[16];
            tmem_ld16(tmem + (lb << 16) + 64u + 32u * pib, o);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(D_O_FREE + pib));
            if (whole) {
                // fold the one split with the sinks here (as decode_fold):
                // M = max(sink log2e, B), L = 2^(sink log2e - M) + l 2^(B - M),
                // out = O 2^(B - M) / L, lse = (M + log2 L) ln 2; the terms are
                // within a factor 2^48 of each other, so the approximate
                // exp2, log2 and reciprocal (relative error ~2^-22) suffice
#pragma unroll
                for (int hh = 0; hh < kGroup; ++hh) {
                    const int h = kGroup * pit.g + hh;
                    const float sink = misc->sinks[h];
                    const float lh = misc->red_l[pib][0][hh] + misc->red_l[pib][1][hh] + misc->red_l[pib][2][hh] +
                                     misc->red_l[pib][3][hh];
                    float ov = 0.f, v;
                    if (sink == INFINITY) {
                        v = INFINITY;
                    } else {
                        const float s2 = sink * 1.4426950408889634f;
                        const float M = fmaxf(s2, B);
                        const float a = dt_ex2(B - M);
                        const float L = (sink > -INFINITY ? dt_ex2(s2 - M) : 0.f) + lh * a;
                        if (L > 0.f) {
                            ov = __uint_as_float(o[hh]) * (a * __frcp_rn(L));
                            v = (M + __log2f(L)) * 0.6931471805599453f;
                        } else {
                            v = -INFINITY;
                        }
                    }
                    p.out[((size_t)pit.b * kHQ + h) * kHD + r] = __float2bfloat16_rn(ov);
                    if (r == 0 && p.lse) p.lse[(size_t)h * p.B + pit.b] = v;
                }
                return true;
            }
#pragma unroll
            for (int h = 0; h < kGroup; ++h) part[2 * kGroup + h * kHD + r] = __uint_as_float(o[h]);
            return finish(pit.b, pit.g);
        };
        bool done = false;                              // the scheduler's end, not a failed wait
        for (;;) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(D_SCHED_FULL + sslot), sph, abort_flag, status))) break;
            const int u = misc->sched[sslot], upos = misc->sched_pos[sslot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(D_SCHED_EMPTY + sslot));
            sslot ^= 1; if (sslot == 0) sph ^= 1;
            if (u < 0) {
                done = true;
                break;
            }
            const DtItem it = dt_item(p, u, upos);
            int nl = 0;
            for (int t = it.t0; t < it.t1; ++t) nl += dt_tile_live(p, it, t) ? 1 : 0;
            if (it.bad && tid == 128) atomicCAS(status, 0, 1 /* FLINT_ERR_INVALID_ARG */);
            if (nl == 0) {
                if (pending && !end_item()) break;
                float* part = part_of(u, it);
                if (warp == 4 && lane < kGroup) { part[lane] = -INFINITY; part[kGroup + lane] = 0.f; }
                if (!finish(it.b, it.g)) break;
                continue;
            }
            const int s_new = it.pos % p.cap;
            // this item's Q^T and new-token scores (query warps)
            const uint32_t ib = k_item & 1u;
            ++k_item;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(D_ITEM_READY + ib), irph[ib], abort_flag, status))) break;
            irph[ib] ^= 1u;
            // ---- the tiles
            float l[kGroup];
#pragma unroll
            for (int h = 0; h < kGroup; ++h) l[h] = 0.f;
            bool alive = true;
            for (int t = it.t0; t < it.t1; ++t) {
                if (!dt_tile_live(p, it, t)) continue;
                const uint32_t sb = tt & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(bar(D_S_FULL + sb), sfph[sb], abort_flag, status))) {
                    alive = false;
                    break;
                }
                sfph[sb] ^= 1u;
                tc_fence_after();
                uint32_t sv[16];
                tmem_ld16(tmem + (lb << 16) + 32u * sb, sv);
                tmem_wait_ld();
                const int slot = t * kDtSlots + r;
                bool valid = slot < p.cap;
                if (valid) {
                    int d = (it.pos - slot) % p.cap;
                    if (d < 0) d += p.cap;
                    valid = d < it.n;
                }
                const bool isnew = slot == s_new;
                float pv[kGroup];
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    const float sc = isnew ? misc->s_new[ib][h] : __uint_as_float(sv[h]) + __uint_as_float(sv[kGroup + h]);
                    pv[h] = valid ? dt_ex2(fmaf(sc, C, -B)) : 0.f;
                    l[h] += pv[h];
                }
                // this P buffer is free once the PV of tile tt - 2 is done
                if (!__all_sync(0xffffffffu, mbar_wait(bar(D_P_FREE + sb), pfph[sb] ^ 1u, abort_flag, status))) {
                    alive = false;
                    break;
                }
                pfph[sb] ^= 1u;
                uint8_t* pbuf = smem + kDtOffP + sb * 2 * kDtB16Half;
#pragma unroll
                for (int h = 0; h < kGroup; ++h)
                    *reinterpret_cast<__nv_bfloat16*>(pbuf + dt_sw_off(h, r, kDtB16Half)) = __float2bfloat16_rn(pv[h]);
                if (isnew) {
                    // the new token's value in its slot row of the V tile
                    uint8_t* vt = smem + sst * kDtStage + kDtTile;
                    const uint4* vsrc = reinterpret_cast<const uint4*>(p.v + ((size_t)it.b * kHKV + it.g) * kHD);
#pragma unroll
                    for (int c8 = 0; c8 < kHD / 8; ++c8)
                        *reinterpret_cast<uint4*>(vt + dt_sw_off(r, 8 * c8, kDtHalf)) = vsrc[c8];
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar(D_P_READY + sb));
                ++tt;
                if (++sst == kDtStages) sst = 0;
                // the previous item's end, now that this item's first tile
                // is with the MMA
                if (pending && !end_item()) {
                    alive = false;
                    break;
                }
            }
            if (!alive) break;
            // the item's Q^T and scores are no longer read: the query warps
            // may fill this parity's buffers for the item after next
            mbar_arrive(bar(D_ITEM_DONE + ib));
            // ---- l over the split's slots, per head: warp sums, then the
            // four warps' sums (read at the item's end)
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                float x = l[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (lane == 0) misc->red_l[ib][wq][h] = x;
            }
            mbar_arrive(bar(D_L_READY));
            if (!__all_sync(0xffffffffu, mbar_wait(bar(D_L_READY), lph, abort_flag, status))) break;
            lph ^= 1;
            pending = true;
            pit = it;
            pu = u;
            pib = ib;
        }
        // the last item's end
        if (done && pending) end_item();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}


// ============================================================================ host
namespace {
bool g_dt_attr[64] = {false};

// 3-D map over a head-major [B, 4, cap, 128] BF16 cache: dims (128, cap,
// B x 4), box (64 channels, 128 slots, one (sequence, KV head)), 128-byte
// swizzle; slots past cap read as zeros.  A tile is two boxes (channel
// halves) of 128 consecutive 256-byte slot rows.
flint_status_t dt_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, int B, int cap) {
    cuuint64_t dims[3] = {(cuuint64_t)kHD, (cuuint64_t)cap, (cuuint64_t)B * kHKV};
    cuuint64_t strides[2] = {(cuuint64_t)kHD * 2, (cuuint64_t)cap * kHD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kDtSlots, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled (decode cache) failed (%d)", (int)r);
    return FLINT_OK;
}
}  // namespace

// Enqueues the tensor-core decode kernel (a no-op when the logit bound is
// above 48) as a programmatic dependent of the kernel that zeroes the status
// word, the unit counter after it and the split-arrival counters.
flint_status_t launch_decode_tc(const DecodeParams& p, int sms, cudaStream_t s) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return fail(FLINT_ERR_UNSUPPORTED, "device index %d", dev);
    if (!g_dt_attr[dev]) {
        cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kDtSmem);
        if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        g_dt_attr[dev] = true;
    }
    EncodeTiledFn enc = nullptr;
    flint_status_t st = get_encoder(&enc);
    if (st != FLINT_OK) return st;
    CUtensorMap tk, tv;
    st = dt_map(enc, &tk, p.k_cache, p.B, p.cap);
    if (st == FLINT_OK) st = dt_map(enc, &tv, p.v_cache, p.B, p.cap);
    if (st != FLINT_OK) return st;
    const long long items = (long long)p.B * kHKV * p.nsplit_tc;
    const int grid = (int)(items < sms ? items : sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDtThreads);
    cfg.dynamicSmemBytes = kDtSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_tc_kernel, tk, tv, p);
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "decode (tensor cores) launch: %s", cudaGetErrorString(e));
    return FLINT_OK;
}

}  // namespace flint
