// backward_tc.cu -- tensor-core (tcgen05 + TMEM + TMA) kernels of the backward
// of one step's chunk SDPA with the step's key set held fixed (bf16 inputs,
// fp32 gradients).
//
// "Learning how to Forget", paper page, section "Gradient Computation
// Strategy for Sparse Attention": training through the sparse cache replays
// the logged eviction decisions, so each step's attention is differentiated
// for the keys it used: the n valid cache slots (visible to every row) and the
// chunk tokens t <= i. With p_ij = exp(scale q_i . k_j - LSE_i),
// dp_ij = dO_i . v_j, D_i = sum_j p_ij dp_ij / sum_j p_ij and
// ds_ij = p_ij (dp_ij - D_i):
//   dq_i = scale sum_j ds_ij k_j,   dk_j = scale sum_i ds_ij q_i,
//   dv_j = sum_i p_ij dO_i
// (sums over i run over every query head of the key's KV group).
//
// bwd_dq_tc_kernel    one CTA per (128-row query tile, head): two passes over
//                     the tile's key blocks. Both compute S = Q K^T and
//                     dP = dO V^T into TMEM; the first only accumulates each
//                     row's sum_j p dp and sum_j p (so D_i is exact in fp32 and
//                     needs no forward output), the second writes
//                     dS = P o (dP - D) to shared memory as a bf16 pair
//                     hi + lo (hi = dS rounded to bf16, lo = the remainder
//                     rounded) and accumulates dQ += hi K + lo K in TMEM: the
//                     terms of dq_i can cancel (equal keys that share a row's
//                     attention), so dS needs more than bf16's 8 bits. It also
//                     writes D_i and the log2-domain LSE per row for the key
//                     kernel.
// bwd_dkdv_tc_kernel  one CTA per (KV group, 128-key block), one key per TMEM
//                     lane: per 128-row query tile of the group's heads,
//                     S^T = K Q^T and dP^T = V dO^T into TMEM, P^T and
//                     dS^T = P^T o (dP^T - D) as bf16 to shared memory, then
//                     dV += P^T dO and dK += dS^T Q in TMEM.
// Both are warp-specialised like the forward kernels: a TMA loader warp, an
// MMA-issuing warp and one 128-thread warpgroup owning one TMEM lane each.
#include <cuda.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace h2o {
namespace {

using tc::desc_kmajor_sw128;
using tc::desc_mnmajor_sw128;
using tc::ex2;
using tc::fence_after_sync;
using tc::fence_before_sync;

struct BwdTcParams {
    int B, Hq, Hkv, T, C, n;
    int n_mblk;    // 128-row query tiles per head
    int nbc;       // cache key blocks = ceil(n / 128)
    int nkb;       // key blocks of cache and chunk
    int rows_pad;  // row stride of the row tables
    float scale_log2, scale;
    const float* lse;  // [B, Hq, T] natural log
    float* Drow;       // [B*Hkv][rows_pad]
    float* L2row;      // [B*Hkv][rows_pad]
    float* dq;         // [B, Hq, T, D]
    float* dKc;        // [B, Hkv, C, D]
    float* dVc;
    float* dk;         // [B, Hkv, T, D]
    float* dv;
    WaitBound wb;
};

// Stores 64 bf16 values (32 packed words) of row r into the 128-byte-swizzled
// K-major half-tile at `half` (rows of 128 bytes, 16-byte chunks XOR-swizzled
// by the row's low three bits), the layout the UMMA descriptors read.
__device__ __forceinline__ void store_row_half(uint8_t* half, int r, const uint32_t (&pk)[32]) {
    uint8_t* row = half + r * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

// ============================================================================
// dQ
// ============================================================================
template <int D>
struct DqCfg {
    static constexpr int HALF = 128 * 128;   // 128 rows x 64 bf16
    static constexpr int TILE = 128 * D * 2;
    static constexpr int RING = 3;           // K / V slots, loaded V0, K0, V1, K1, ...
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_DO = TILE;
    static constexpr int OFF_RING = 2 * TILE;
    static constexpr int OFF_DS = OFF_RING + RING * TILE;  // dS hi tile, two halves of 64 keys
    static constexpr int OFF_DSL = OFF_DS + 2 * HALF;     // dS lo tile
    static constexpr int OFF_BAR = OFF_DSL + 2 * HALF;
    static constexpr int NBAR = 20;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
    static constexpr int THREADS = 192;      // loader, MMA, one warpgroup
    static constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_DQ = tc::idesc_bf16_f32(128, D, true);
};
static_assert(DqCfg<128>::SMEM <= 232448, "dQ kernel shared memory exceeds the per-CTA limit");

template <int D>
__global__ void __launch_bounds__(DqCfg<D>::THREADS, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                 const __grid_constant__ CUtensorMap map_kc, const __grid_constant__ CUtensorMap map_vc,
                 const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                 const BwdTcParams p) {
    using Cfg = DqCfg<D>;
    constexpr int RING = Cfg::RING;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* q_full = bars;                 // Q and dO tiles
    uint64_t* ring_full = bars + 1;          // [RING]
    uint64_t* ring_empty = ring_full + RING; // [RING]
    uint64_t* s_full = ring_empty + RING;    // S and dP in TMEM
    uint64_t* s_free = s_full + 1;           // 4 arrivals: S and dP in registers
    uint64_t* ds_full = s_free + 1;          // [2 halves], 4 arrivals
    uint64_t* ds_done = ds_full + 2;         // [2 halves]: dQ MMAs of that half completed
    uint64_t* drain = ds_done + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int G = p.Hq / p.Hkv;
    const int per_mblk = p.B * p.Hq;
    const int mblk = p.n_mblk - 1 - (int)(blockIdx.x / per_mblk);  // most key blocks first
    const int bh = blockIdx.x % per_mblk;
    const int b = bh / p.Hq, h = bh % p.Hq;
    const int bg = b * p.Hkv + h / G;
    const int m0 = mblk * 128;
    const int nb = p.nbc + mblk + 1;  // key blocks per pass: cache, then chunk 0..mblk
    const int iters = 2 * nb;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < RING; ++s) {
            mbar_init(ring_full + s, 1);
            mbar_init(ring_empty + s, 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 4);
        for (int hh = 0; hh < 2; ++hh) {
            mbar_init(ds_full + hh, 4);
            mbar_init(ds_done + hh, 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;  // S at 0, dP at 128, dQ at 256
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            tc::prefetch_tmap(&map_q);
            tc::prefetch_tmap(&map_do);
            const int qrow = (b * p.Hq + h) * p.T + m0;
            mbar_arrive_expect_tx(q_full, 2 * Cfg::TILE);
            for (int hh = 0; hh < D / 64; ++hh) {
                tc::tma_load_2d(smem + Cfg::OFF_Q + hh * Cfg::HALF, &map_q, 64 * hh, qrow, q_full);
                tc::tma_load_2d(smem + Cfg::OFF_DO + hh * Cfg::HALF, &map_do, 64 * hh, qrow, q_full);
            }
            int L = 0;
            bool ok = true;
            for (int it = 0; ok && it < iters; ++it) {
                const int j = it % nb;
                const bool cache = j < p.nbc;
                const int row = cache ? bg * p.C + 128 * j : bg * p.T + 128 * (j - p.nbc);
                // V before K: V(j+1) then reuses the slot of K(j-1), K(j+1) that of
                // V(j), and both are released early in the block
                for (int kv = 0; ok && kv < 2; ++kv, ++L) {
                    const int slot = L % RING;
                    if (!(ok = wait_bar(ring_empty + slot, ((L / RING) & 1) ^ 1, p.wb, kDevTimeoutSlotWait,
                                        abort_flag)))
                        break;
                    const CUtensorMap* map = kv ? (cache ? &map_kc : &map_k) : (cache ? &map_vc : &map_v);
                    mbar_arrive_expect_tx(ring_full + slot, Cfg::TILE);
                    for (int hh = 0; hh < D / 64; ++hh)
                        tc::tma_load_2d(smem + Cfg::OFF_RING + slot * Cfg::TILE + hh * Cfg::HALF, map, 64 * hh, row,
                                        ring_full + slot);
                }
            }
            wait_bar(q_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
            for (int s = 0; s < RING; ++s) {
                const int uses = L / RING + (s < L % RING ? 1 : 0);
                if (uses) wait_bar(ring_full + s, (uses - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t dQd = desc_kmajor_sw128(sbase + Cfg::OFF_Q);
        const uint64_t dOd = desc_kmajor_sw128(sbase + Cfg::OFF_DO);
        const uint64_t dRingK = desc_kmajor_sw128(sbase + Cfg::OFF_RING);
        const uint64_t dRingN = desc_mnmajor_sw128(sbase + Cfg::OFF_RING, Cfg::HALF);
        const uint64_t dDS = desc_kmajor_sw128(sbase + Cfg::OFF_DS);
        const uint64_t dDSL = desc_kmajor_sw128(sbase + Cfg::OFF_DSL);
        int L = 0;
        bool ok = warp_wait(q_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
        for (int it = 0; ok && it < iters; ++it) {
            const bool pass2 = it >= nb;
            const int j = it - (pass2 ? nb : 0);
            const int vs = L % RING, vu = L / RING;
            const int ks = (L + 1) % RING, ku = (L + 1) / RING;
            L += 2;
            ok = warp_wait(ring_full + ks, ku & 1, p.wb, kDevTimeoutTmaWait, abort_flag) &&
                 warp_wait(ring_full + vs, vu & 1, p.wb, kDevTimeoutTmaWait, abort_flag) &&
                 (it == 0 || warp_wait(s_free, (it - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag));
            if (!ok) break;
            fence_after_sync();
            if (lane == 0) {
                const uint64_t dK = dRingK + (uint64_t)((ks * Cfg::TILE) >> 4);
                const uint64_t dV = dRingK + (uint64_t)((vs * Cfg::TILE) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Cfg::HALF + (kk & 3) * 32) >> 4;
                    tc::mma_bf16_ss(tmem, dQd + off, dK + off, Cfg::IDESC_S, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Cfg::HALF + (kk & 3) * 32) >> 4;
                    tc::mma_bf16_ss(tmem + 128, dOd + off, dV + off, Cfg::IDESC_S, kk > 0);
                }
                tc::mma_commit(s_full);
                tc::mma_commit(ring_empty + vs);
                if (!pass2) tc::mma_commit(ring_empty + ks);
            }
            __syncwarp();
            if (pass2) {
                // dQ += (dS hi + dS lo) K, one 64-key half at a time (K as the
                // N-contiguous B operand)
                for (int hh = 0; hh < 2; ++hh) {
                    if (!(ok = warp_wait(ds_full + hh, j & 1, p.wb, kDevTimeoutMmaWait, abort_flag))) break;
                    fence_after_sync();
                    if (lane == 0) {
                        const uint64_t dKn = dRingN + (uint64_t)((ks * Cfg::TILE) >> 4);
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int kk = 4 * hh + k4;
                            const uint64_t aoff = (uint64_t)((hh * Cfg::HALF + k4 * 32) >> 4);
                            const uint64_t boff = (uint64_t)((kk * 16 * 128) >> 4);
                            tc::mma_bf16_ss(tmem + 256, dDS + aoff, dKn + boff, Cfg::IDESC_DQ, (j > 0 || kk > 0) ? 1u : 0u);
                            tc::mma_bf16_ss(tmem + 256, dDSL + aoff, dKn + boff, Cfg::IDESC_DQ, 1u);
                        }
                        tc::mma_commit(ds_done + hh);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) tc::mma_commit(ring_empty + ks);
                __syncwarp();
            }
        }
        if (lane == 0) tc::mma_commit(drain);
        __syncwarp();
        warp_wait(drain, 0, p.wb, kDevTimeoutMmaWait, abort_flag);
    } else {
        // --------------------------------------------------------- row warpgroup
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // row inside the tile = TMEM lane
        const int i = m0 + r;
        const bool row_ok = i < p.T;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float L2 = row_ok ? p.lse[(size_t)(b * p.Hq + h) * p.T + i] * kLog2e : 0.f;
        float Dacc = 0.f, Pacc = 0.f, Dfin = 0.f;
        bool ok = true;
        for (int it = 0; it < iters; ++it) {
            const bool pass2 = it >= nb;
            const int j = it - (pass2 ? nb : 0);
            if (!(ok = warp_wait(s_full, it & 1, p.wb, kDevTimeoutMmaWait, abort_flag))) break;
            fence_after_sync();
            // visible columns of this row in block j: col < limit
            const int limit = !row_ok ? 0 : (j < p.nbc) ? p.n - 128 * j : i - 128 * (j - p.nbc) + 1;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t s[2][32], dp[2][32];
                tc::tmem_ld32(tmem + lane_off + 64 * hf, s[0]);
                tc::tmem_ld32(tmem + lane_off + 64 * hf + 32, s[1]);
                tc::tmem_ld32(tmem + 128 + lane_off + 64 * hf, dp[0]);
                tc::tmem_ld32(tmem + 128 + lane_off + 64 * hf + 32, dp[1]);
                tc::tmem_ld_wait();
                if (hf == 1) {
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_free);
                }
                uint32_t pk[32], pl[32];
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    const int col = 64 * hf + e;
                    float p0 = ex2(fmaf(__uint_as_float(s[e >> 5][e & 31]), p.scale_log2, -L2));
                    float p1 = ex2(fmaf(__uint_as_float(s[e >> 5][(e & 31) + 1]), p.scale_log2, -L2));
                    p0 = col < limit ? p0 : 0.f;
                    p1 = col + 1 < limit ? p1 : 0.f;
                    const float dp0 = __uint_as_float(dp[e >> 5][e & 31]);
                    const float dp1 = __uint_as_float(dp[e >> 5][(e & 31) + 1]);
                    if (!pass2) {
                        Dacc = fmaf(p0, dp0, fmaf(p1, dp1, Dacc));
                        Pacc += p0 + p1;
                    } else {
                        const float ds0 = p0 * (dp0 - Dfin), ds1 = p1 * (dp1 - Dfin);
                        const uint32_t hi = tc::pack_bf16(ds0, ds1);
                        pk[e >> 1] = hi;
                        pl[e >> 1] = tc::pack_bf16(ds0 - __uint_as_float(hi << 16), ds1 - __uint_as_float(hi & 0xffff0000u));
                    }
                }
                if (pass2) {
                    // the half's buffer is free once the dQ MMAs of block j-1 read it
                    if (j > 0 && ok) ok = warp_wait(ds_done + hf, (j - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
                    store_row_half(smem + Cfg::OFF_DS + hf * Cfg::HALF, r, pk);
                    store_row_half(smem + Cfg::OFF_DSL + hf * Cfg::HALF, r, pl);
                    tc::fence_proxy_async_smem();
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ds_full + hf);
                }
            }
            if (!ok) break;
            if (it == nb - 1) {
                // end of the first pass: the row term, for the second pass and
                // for the key kernel (every valid row sees at least one key)
                Dfin = row_ok ? Dacc / Pacc : 0.f;
                if (row_ok) {
                    const size_t ro = (size_t)bg * p.rows_pad + (size_t)(h % G) * p.T + i;
                    p.Drow[ro] = Dfin;
                    p.L2row[ro] = L2;
                }
            }
        }
        // ------------------------------------------------------------ epilogue
        if (ok && warp_wait(ds_done + 1, (nb - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag)) {
            fence_after_sync();
            float* drow = p.dq + ((size_t)(b * p.Hq + h) * p.T + i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tmem + 256 + lane_off + 32 * c, o);
                tc::tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        *reinterpret_cast<float4*>(drow + 32 * c + 4 * q4) =
                            make_float4(__uint_as_float(o[4 * q4]) * p.scale, __uint_as_float(o[4 * q4 + 1]) * p.scale,
                                        __uint_as_float(o[4 * q4 + 2]) * p.scale,
                                        __uint_as_float(o[4 * q4 + 3]) * p.scale);
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ============================================================================
// dK, dV
// ============================================================================
template <int D>
struct DkvCfg {
    static constexpr int HALF = 128 * 128;   // 128 rows x 64 bf16
    static constexpr int TILE = 128 * D * 2;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = TILE;
    static constexpr int OFF_Q = 2 * TILE;
    static constexpr int OFF_DO = 3 * TILE;
    static constexpr int OFF_P = 4 * TILE;         // P^T, two halves of 64 rows
    static constexpr int OFF_DS = OFF_P + 2 * HALF; // dS^T, two halves
    static constexpr int OFF_ROWT = OFF_DS + 2 * HALF;  // [2][2][128] floats: -L2 and D per tile row
    static constexpr int OFF_BAR = OFF_ROWT + 2 * 2 * 128 * 4;
    static constexpr int NBAR = 16;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
    static constexpr int THREADS = 192;
    static constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_G = tc::idesc_bf16_f32(128, D, true);
};
static_assert(DkvCfg<128>::SMEM <= 232448, "dK/dV kernel shared memory exceeds the per-CTA limit");

template <int D>
__global__ void __launch_bounds__(DkvCfg<D>::THREADS, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                   const __grid_constant__ CUtensorMap map_kc, const __grid_constant__ CUtensorMap map_vc,
                   const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                   const BwdTcParams p) {
    using Cfg = DkvCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* kv_full = bars;        // the key block's K and V
    uint64_t* t_full = bars + 1;     // a query tile's Q and dO
    uint64_t* t_empty = bars + 2;    // its MMAs have completed
    uint64_t* s_full = bars + 3;     // S^T and dP^T in TMEM
    uint64_t* s_free = bars + 4;     // 4 arrivals: in registers
    uint64_t* pt_full = bars + 5;    // [2 halves], 4 arrivals: P^T and dS^T half written
    uint64_t* pt_done = bars + 7;    // [2 halves]: dV / dK MMAs of that half completed
    uint64_t* drain = bars + 9;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int G = p.Hq / p.Hkv;
    const int groups = p.B * p.Hkv;
    const int kb = blockIdx.x / groups;  // cache blocks (all rows see them) first
    const int bg = blockIdx.x % groups;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const bool cache = kb < p.nbc;
    const int t0 = cache ? 0 : 128 * (kb - p.nbc);  // first chunk token of the block
    const int n_keys = cache ? min(128, p.n - 128 * kb) : min(128, p.T - t0);
    const int key_row = cache ? bg * p.C + 128 * kb : bg * p.T + t0;
    const int m_first = cache ? 0 : t0 / 128;  // query tiles before it cannot see a chunk block
    const int tiles_per_head = p.n_mblk - m_first;
    const int ntiles = G * tiles_per_head;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(t_full, 1);
        mbar_init(t_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(s_free, 4);
        for (int hh = 0; hh < 2; ++hh) {
            mbar_init(pt_full + hh, 4);
            mbar_init(pt_done + hh, 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;  // S^T at 0, dP^T at 128, dV at 256, dK at 256 + D
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            tc::prefetch_tmap(&map_q);
            tc::prefetch_tmap(&map_do);
            mbar_arrive_expect_tx(kv_full, 2 * Cfg::TILE);
            for (int hh = 0; hh < D / 64; ++hh) {
                tc::tma_load_2d(smem + Cfg::OFF_K + hh * Cfg::HALF, cache ? &map_kc : &map_k, 64 * hh, key_row,
                                kv_full);
                tc::tma_load_2d(smem + Cfg::OFF_V + hh * Cfg::HALF, cache ? &map_vc : &map_v, 64 * hh, key_row,
                                kv_full);
            }
            int loaded = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int hh = t / tiles_per_head, m = m_first + t % tiles_per_head;
                if (!wait_bar(t_empty, (t & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag)) break;
                const int qrow = (b * p.Hq + g * G + hh) * p.T + 128 * m;
                mbar_arrive_expect_tx(t_full, 2 * Cfg::TILE);
                for (int x = 0; x < D / 64; ++x) {
                    tc::tma_load_2d(smem + Cfg::OFF_Q + x * Cfg::HALF, &map_q, 64 * x, qrow, t_full);
                    tc::tma_load_2d(smem + Cfg::OFF_DO + x * Cfg::HALF, &map_do, 64 * x, qrow, t_full);
                }
                ++loaded;
            }
            wait_bar(kv_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
            if (loaded) wait_bar(t_full, (loaded - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t dK = desc_kmajor_sw128(sbase + Cfg::OFF_K);
        const uint64_t dV = desc_kmajor_sw128(sbase + Cfg::OFF_V);
        const uint64_t dQk = desc_kmajor_sw128(sbase + Cfg::OFF_Q);
        const uint64_t dOk = desc_kmajor_sw128(sbase + Cfg::OFF_DO);
        const uint64_t dQn = desc_mnmajor_sw128(sbase + Cfg::OFF_Q, Cfg::HALF);
        const uint64_t dOn = desc_mnmajor_sw128(sbase + Cfg::OFF_DO, Cfg::HALF);
        const uint64_t dP = desc_kmajor_sw128(sbase + Cfg::OFF_P);
        const uint64_t dS = desc_kmajor_sw128(sbase + Cfg::OFF_DS);
        bool ok = warp_wait(kv_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
        for (int t = 0; ok && t < ntiles; ++t) {
            ok = warp_wait(t_full, t & 1, p.wb, kDevTimeoutTmaWait, abort_flag) &&
                 (t == 0 || warp_wait(s_free, (t - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag));
            if (!ok) break;
            fence_after_sync();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Cfg::HALF + (kk & 3) * 32) >> 4;
                    tc::mma_bf16_ss(tmem, dK + off, dQk + off, Cfg::IDESC_S, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Cfg::HALF + (kk & 3) * 32) >> 4;
                    tc::mma_bf16_ss(tmem + 128, dV + off, dOk + off, Cfg::IDESC_S, kk > 0);
                }
                tc::mma_commit(s_full);
            }
            __syncwarp();
            // dV += P^T dO and dK += dS^T Q, one 64-row half of the tile at a time
            for (int hh = 0; hh < 2; ++hh) {
                if (!(ok = warp_wait(pt_full + hh, t & 1, p.wb, kDevTimeoutMmaWait, abort_flag))) break;
                fence_after_sync();
                if (lane == 0) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = 4 * hh + k4;
                        const uint64_t aoff = (uint64_t)((hh * Cfg::HALF + k4 * 32) >> 4);
                        const uint64_t boff = (uint64_t)((kk * 16 * 128) >> 4);
                        const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                        tc::mma_bf16_ss(tmem + 256, dP + aoff, dOn + boff, Cfg::IDESC_G, acc);
                        tc::mma_bf16_ss(tmem + 256 + D, dS + aoff, dQn + boff, Cfg::IDESC_G, acc);
                    }
                    tc::mma_commit(pt_done + hh);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) tc::mma_commit(t_empty);
            __syncwarp();
        }
        if (lane == 0) tc::mma_commit(drain);
        __syncwarp();
        warp_wait(drain, 0, p.wb, kDevTimeoutMmaWait, abort_flag);
    } else {
        // --------------------------------------------------------- key warpgroup
        const int quad = warp & 3;
        const int kr = quad * 32 + lane;  // key inside the block = TMEM lane
        const bool key_ok = kr < n_keys;
        const int t_key = cache ? -1 : t0 + kr;  // chunk token index of this key
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float* rowt = reinterpret_cast<float*>(smem + Cfg::OFF_ROWT);
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            const int hh = t / tiles_per_head, m = m_first + t % tiles_per_head;
            // this tile's row terms: -L2 and D per row, staged by the 128 threads
            float* rt = rowt + (t & 1) * 256;
            {
                const int i = 128 * m + kr;
                const size_t ro = (size_t)bg * p.rows_pad + (size_t)hh * p.T + (i < p.T ? i : 0);
                rt[kr] = i < p.T ? -p.L2row[ro] : 0.f;
                rt[128 + kr] = i < p.T ? p.Drow[ro] : 0.f;
            }
            tc::named_sync(1, 128);
            if (ok) ok = warp_wait(s_full, t & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
            if (!ok) continue;  // keep joining the named barrier until the loop ends
            fence_after_sync();
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t s[2][32], dp[2][32];
                tc::tmem_ld32(tmem + lane_off + 64 * hf, s[0]);
                tc::tmem_ld32(tmem + lane_off + 64 * hf + 32, s[1]);
                tc::tmem_ld32(tmem + 128 + lane_off + 64 * hf, dp[0]);
                tc::tmem_ld32(tmem + 128 + lane_off + 64 * hf + 32, dp[1]);
                tc::tmem_ld_wait();
                if (hf == 1) {
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_free);
                }
                uint32_t pp[32], pd[32];
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    const int c = 64 * hf + e;        // column = query row 128 m + c
                    const int i = 128 * m + c;
                    const bool v0 = key_ok && i < p.T && i >= t_key;
                    const bool v1 = key_ok && i + 1 < p.T && i + 1 >= t_key;
                    float p0 = ex2(fmaf(__uint_as_float(s[e >> 5][e & 31]), p.scale_log2, rt[c]));
                    float p1 = ex2(fmaf(__uint_as_float(s[e >> 5][(e & 31) + 1]), p.scale_log2, rt[c + 1]));
                    p0 = v0 ? p0 : 0.f;
                    p1 = v1 ? p1 : 0.f;
                    const float ds0 = p0 * (__uint_as_float(dp[e >> 5][e & 31]) - rt[128 + c]);
                    const float ds1 = p1 * (__uint_as_float(dp[e >> 5][(e & 31) + 1]) - rt[128 + c + 1]);
                    pp[e >> 1] = tc::pack_bf16(p0, p1);
                    pd[e >> 1] = tc::pack_bf16(ds0, ds1);
                }
                // the halves are free once the MMAs of tile t-1 read them
                if (t > 0 && ok) ok = warp_wait(pt_done + hf, (t - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
                store_row_half(smem + Cfg::OFF_P + hf * Cfg::HALF, kr, pp);
                store_row_half(smem + Cfg::OFF_DS + hf * Cfg::HALF, kr, pd);
                tc::fence_proxy_async_smem();
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(pt_full + hf);
            }
        }
        // ------------------------------------------------------------ epilogue
        if (ok && ntiles > 0 && warp_wait(pt_done + 1, (ntiles - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag)) {
            fence_after_sync();
            float* gv = cache ? p.dVc + ((size_t)bg * p.C + 128 * kb + kr) * D
                              : p.dv + ((size_t)bg * p.T + t0 + kr) * D;
            float* gk = cache ? p.dKc + ((size_t)bg * p.C + 128 * kb + kr) * D
                              : p.dk + ((size_t)bg * p.T + t0 + kr) * D;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float* dst = part ? gk : gv;
                const float mul = part ? p.scale : 1.f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tc::tmem_ld32(tmem + 256 + part * D + lane_off + 32 * c, o);
                    tc::tmem_ld_wait();
                    if (key_ok) {
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            *reinterpret_cast<float4*>(dst + 32 * c + 4 * q4) =
                                make_float4(__uint_as_float(o[4 * q4]) * mul, __uint_as_float(o[4 * q4 + 1]) * mul,
                                            __uint_as_float(o[4 * q4 + 2]) * mul,
                                            __uint_as_float(o[4 * q4 + 3]) * mul);
                    }
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t backward_launch(const BwdArgs& a) {
    if (cudaError_t e = ensure_smem_limit(bwd_dq_tc_kernel<D>, DqCfg<D>::SMEM); e != cudaSuccess) return e;
    if (cudaError_t e = ensure_smem_limit(bwd_dkdv_tc_kernel<D>, DkvCfg<D>::SMEM); e != cudaSuccess) return e;
    CUtensorMap mq, mdo, mkc, mvc, mk, mv;
    const uint64_t qrows = (uint64_t)a.B * a.Hq * a.T;
    if (!tc_make_map(&mq, a.q, qrows, D, 128) || !tc_make_map(&mdo, a.dout, qrows, D, 128) ||
        !tc_make_map(&mkc, a.Kc, (uint64_t)a.B * a.Hkv * a.C, D, 128) ||
        !tc_make_map(&mvc, a.Vc, (uint64_t)a.B * a.Hkv * a.C, D, 128) ||
        !tc_make_map(&mk, a.k, (uint64_t)a.B * a.Hkv * a.T, D, 128) ||
        !tc_make_map(&mv, a.v, (uint64_t)a.B * a.Hkv * a.T, D, 128))
        return cudaErrorInvalidValue;
    BwdTcParams p;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.T = a.T;
    p.C = a.C;
    p.n = a.n;
    p.n_mblk = (a.T + 127) / 128;
    p.nbc = (a.n + 127) / 128;
    p.nkb = p.nbc + p.n_mblk;
    p.rows_pad = a.rows_pad;
    p.scale = 1.f / sqrtf((float)D);
    p.scale_log2 = kLog2e * p.scale;
    p.lse = a.lse;
    p.Drow = a.Drow;
    p.L2row = a.L2row;
    p.dq = a.dq;
    p.dKc = a.dKc;
    p.dVc = a.dVc;
    p.dk = a.dk;
    p.dv = a.dv;
    p.wb = a.wb;
    // empty cache slots get zero gradients (the key kernel writes only valid keys)
    if (a.n < a.C) {
        const size_t pitch = (size_t)a.C * D * sizeof(float);
        const size_t width = (size_t)(a.C - a.n) * D * sizeof(float);
        const size_t off = (size_t)a.n * D;
        cudaError_t e = cudaMemset2DAsync(a.dKc + off, pitch, 0, width, (size_t)a.B * a.Hkv, a.stream);
        if (e == cudaSuccess) e = cudaMemset2DAsync(a.dVc + off, pitch, 0, width, (size_t)a.B * a.Hkv, a.stream);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_ex(false, bwd_dq_tc_kernel<D>, dim3(p.n_mblk * a.B * a.Hq), dim3(DqCfg<D>::THREADS),
                              DqCfg<D>::SMEM, a.stream, mq, mdo, mkc, mvc, mk, mv, p);
    if (e != cudaSuccess) return e;
    a.log->done("bwd_dq_tc_kernel", a.stream);
    e = launch_ex(false, bwd_dkdv_tc_kernel<D>, dim3(p.nkb * a.B * a.Hkv), dim3(DkvCfg<D>::THREADS),
                  DkvCfg<D>::SMEM, a.stream, mq, mdo, mkc, mvc, mk, mv, p);
    if (e != cudaSuccess) return e;
    a.log->done("bwd_dkdv_tc_kernel", a.stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t tc_backward(const BwdArgs& a) { return a.d == 64 ? backward_launch<64>(a) : backward_launch<128>(a); }

}  // namespace h2o
