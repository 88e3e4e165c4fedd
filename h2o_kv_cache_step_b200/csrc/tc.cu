// tc.cu -- tensor-core (tcgen05 + TMEM + TMA) kernels of the bf16 H2O step.
//
// sdpa_tc_kernel   chunk SDPA ("Learning how to Forget", paper page, section
//                  "Kernel Support Needs": SDPA under the positional mask):
//                  O = softmax(scale * Q K^T) V over the n cache slots plus the
//                  chunk tokens t <= i, and each row's log-sum-exp.
// wsum_tc_kernel   the summed attention weights the same section asks kernels
//                  to return, per key: sum over query rows i (and the query
//                  heads of its KV group) of exp(scale * q_i . k - LSE_i);
//                  the paper page's section "Improvements to Heavy-Hitter
//                  Oracle (H2O)" adds them to the H2O scores.
//
// Both are warp-specialised, one CTA = 6 warps:
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM owner and tcgen05.mma issuer (one elected lane)
//   warps 2..5  128 threads, one TMEM lane (matrix row) each
//
// SDPA: M = 128 query rows of one head, N = 128 keys per block, K = d.
//   S = Q K^T goes to one of two TMEM buffers; the softmax warps turn it into
//   P (bf16, written to shared memory in the 128-byte-swizzled K-major layout
//   the next MMA reads) and O += P V accumulates in TMEM. The running maximum
//   is only moved (and O rescaled in TMEM) when it grows by more than 2^8,
//   so P stays below 256 and most blocks skip the rescale.
// Weight sums: the transposed product S^T = K Q^T puts one KEY on each TMEM
//   lane (M = 128 keys) and 128 query rows on the columns, so each thread sums
//   its own key's weights across the columns in registers: the reduction over
//   queries needs no shuffles and no atomics. Query rows are split into parts
//   (per-CTA partials); the selection kernel adds the parts in a fixed order.
#include <cuda.h>

#include <mutex>

#include "tc.h"
#include "tc_ptx.cuh"

namespace h2o {
namespace {

using tc::desc_kmajor_sw128;
using tc::desc_mnmajor_sw128;
using tc::ex2;
using tc::fence_after_sync;
using tc::fence_before_sync;

constexpr int kThreads = 192;
constexpr int kRowsPerPart = 1024;   // weight-sum rows per CTA (8 tiles of 128)
constexpr float kRescaleThreshold = 8.f;  // log2 units
// Of every 8 columns, how many take the FMA-pipe exp2 instead of the MUFU
// unit (the MUFU is the other bottleneck next to the tensor core).
#ifndef H2O_POLY_SDPA
#define H2O_POLY_SDPA 1
#endif
#ifndef H2O_POLY_WSUM
#define H2O_POLY_WSUM 2
#endif
constexpr int kPolyPairsOf4Sdpa = H2O_POLY_SDPA;  // SDPA: pairs in every 4 on the FMA pipe
constexpr int kPolyPairsOf8Wsum = H2O_POLY_WSUM;  // weight sums: pairs in every 8 on the FMA pipe

// Bounded wait that also gives up once another role has given up.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const WaitBound& wb, int code,
                                         volatile int* abort_flag) {
    const uint32_t addr = smem_u32(bar);
    if (mbar_try_wait(addr, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        for (int i = 0; i < 8; ++i)
            if (mbar_try_wait_sleep(addr, parity, 20000u)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > wb.ns) {
            record_error(wb, code);
            *abort_flag = 1;
            return false;
        }
    }
}

// Every lane waits; the outcome is made warp-uniform so that a give-up never
// leaves part of a warp behind at a warp-collective instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitBound& wb, int code,
                                          volatile int* abort_flag) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, wb, code, abort_flag));
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

// ============================================================================
// SDPA
// ============================================================================
// Two CTAs share an SM: each holds Q (one 128-row tile), one K block and one
// V block in shared memory, and 256 TMEM columns: S (128 fp32 columns; P, bf16
// packed two per column, overwrites its first 64 after the softmax has read
// them) and O (d columns). A CTA's own chain QK(j) -> softmax(j) -> PV(j) ->
// QK(j+1) is serial; the other CTA's MMAs fill the tensor core meanwhile.
template <int D>
struct SdpaCfg {
    static constexpr int HALF = 128 * 128;       // bytes of one 128-row x 64-col bf16 box
    static constexpr int TILE = 128 * D * 2;     // one 128-row x d tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;
    static constexpr int OFF_V = 2 * TILE;
    static constexpr int OFF_BAR = 3 * TILE;
    static constexpr int NBAR = 12;
    static constexpr int SMEM_RAW = OFF_BAR + NBAR * 8 + 16 + 1024;
    // at least ~80 KB so that no more than two CTAs (2 x 256 TMEM columns)
    // share an SM
    static constexpr int SMEM = SMEM_RAW > 80 * 1024 ? SMEM_RAW : 80 * 1024;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t IDESC_QK = tc::idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(128, D, true);
};

struct SdpaParams {
    int B, Hq, Hkv, T, C, n, tmax;
    int n_mblk;   // query-row tiles per head
    int nbc;      // cache key blocks = ceil(n / 128)
    float scale_log2;
    __nv_bfloat16* out;
    float* lse;
    WaitBound wb;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
sdpa_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
               const __grid_constant__ CUtensorMap map_vc, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_v, const SdpaParams p) {
    using Cfg = SdpaCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = bars + 2;
    uint64_t* v_full = bars + 3;
    uint64_t* v_empty = bars + 4;
    uint64_t* s_full = bars + 5;
    uint64_t* p_full = bars + 6;
    uint64_t* pv_done = bars + 7;
    uint64_t* drain = bars + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // Tiles in decreasing amount of work: the last query-row tile of each head
    // sees the most chunk keys, so tiles are issued from the last one down.
    const int BH = p.B * p.Hq;
    const int mblk = p.n_mblk - 1 - (int)(blockIdx.x / BH);
    const int bh = blockIdx.x % BH;
    const int b = bh / p.Hq, h = bh % p.Hq;
    const int G = p.Hq / p.Hkv;
    const int bg = b * p.Hkv + h / G;
    const int m0 = mblk * 128;
    const int nb = p.nbc + mblk + 1;  // cache blocks, then chunk blocks 0..mblk

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(k_full, 1);
        mbar_init(k_empty, 1);
        mbar_init(v_full, 1);
        mbar_init(v_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 128;

    const uint32_t sbase = smem_u32(smem);
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::prefetch_tmap(&map_q);
            tc::prefetch_tmap(&map_kc);
            tc::prefetch_tmap(&map_k);
            int nk = 0, nv = 0;
            mbar_arrive_expect_tx(q_full, Cfg::TILE);
            const int qrow = (b * p.Hq + h) * p.T + m0;
            for (int hh = 0; hh < D / 64; ++hh)
                tc::tma_load_2d(smem + Cfg::OFF_Q + hh * Cfg::HALF, &map_q, 64 * hh, qrow, q_full);
            for (int j = 0; j < nb; ++j) {
                const bool cache = j < p.nbc;
                const CUtensorMap* mk = cache ? &map_kc : &map_k;
                const CUtensorMap* mv = cache ? &map_vc : &map_v;
                const int row = cache ? bg * p.C + 128 * j : bg * p.T + 128 * (j - p.nbc);
                // K(j) once QK(j-1) has read K(j-1)
                if (!wait_bar(k_empty, (j & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag)) break;
                mbar_arrive_expect_tx(k_full, Cfg::TILE);
                for (int hh = 0; hh < D / 64; ++hh)
                    tc::tma_load_2d(smem + Cfg::OFF_K + hh * Cfg::HALF, mk, 64 * hh, row, k_full);
                ++nk;
                // V(j) once PV(j-1) has read V(j-1)
                if (!wait_bar(v_empty, (j & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag)) break;
                mbar_arrive_expect_tx(v_full, Cfg::TILE);
                for (int hh = 0; hh < D / 64; ++hh)
                    tc::tma_load_2d(smem + Cfg::OFF_V + hh * Cfg::HALF, mv, 64 * hh, row, v_full);
                ++nv;
            }
            // every load issued here has landed before the CTA may exit
            wait_bar(q_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
            if (nk) wait_bar(k_full, (nk - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
            if (nv) wait_bar(v_full, (nv - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------- MMA issuer
        bool ok = warp_wait(q_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
        const uint32_t sQ = sbase + Cfg::OFF_Q, sK = sbase + Cfg::OFF_K, sV = sbase + Cfg::OFF_V;
        for (int j = 0; ok && j < nb; ++j) {
            // S/P columns are free (and O stable) once PV(j-1) has completed
            ok = warp_wait(k_full, j & 1, p.wb, kDevTimeoutTmaWait, abort_flag) &&
                 (j == 0 || warp_wait(pv_done, (j - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag));
            if (!ok) break;
            fence_after_sync();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * Cfg::HALF + (kk & 3) * 32;
                    tc::mma_bf16_ss(tS, desc_kmajor_sw128(sQ + off), desc_kmajor_sw128(sK + off), Cfg::IDESC_QK,
                                    kk > 0);
                }
                tc::mma_commit(s_full);
                tc::mma_commit(k_empty);
            }
            __syncwarp();
            ok = warp_wait(p_full, j & 1, p.wb, kDevTimeoutMmaWait, abort_flag) &&
                 warp_wait(v_full, j & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
            if (!ok) break;
            fence_after_sync();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // 128 keys, 16 per instruction
                    tc::mma_bf16_ts(tO, tS + 8 * kk, desc_mnmajor_sw128(sV + kk * 16 * 128, Cfg::HALF),
                                    Cfg::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(pv_done);
                tc::mma_commit(v_empty);
            }
            __syncwarp();
        }
        // all MMAs issued here complete before TMEM can be released
        if (lane == 0) tc::mma_commit(drain);
        __syncwarp();
        warp_wait(drain, 0, p.wb, kDevTimeoutMmaWait, abort_flag);
    } else {
        // -------------------------------------------------------------- softmax
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // row inside the tile = TMEM lane
        const int i = m0 + r;            // query row inside the chunk
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
            ok = warp_wait(s_full, j & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
            if (!ok) break;
            fence_after_sync();
            // visible columns of this row in block j: col < limit
            int limit;
            if (j < p.nbc) {
                limit = p.n - 128 * j;
            } else {
                limit = min(i, p.T - 1) - 128 * (j - p.nbc) + 1;
            }
            // pass 1: maximum of the raw visible scores (the scale is positive)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(tS + lane_off + 32 * c, v);
                tc::tmem_ld_wait();
                if (limit >= 128) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        mx0 = tc::max3(mx0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        mx1 = tc::max3(mx1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float a0 = (32 * c + e < limit) ? __uint_as_float(v[e]) : -INFINITY;
                        const float a1 = (32 * c + e + 1 < limit) ? __uint_as_float(v[e + 1]) : -INFINITY;
                        mx0 = tc::max3(mx0, a0, a1);
                    }
                }
            }
            const float m_new = fmaxf(m_run, fmaxf(mx0, mx1) * p.scale_log2);
            const bool resc = m_new > m_run + kRescaleThreshold;
            const float m_use = resc ? m_new : m_run;
            const float alpha = resc ? ex2(m_run - m_use) : 1.f;
            const float msub = (m_use == -INFINITY) ? 0.f : m_use;
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                // O is stable: QK(j) was only issued after PV(j-1) completed
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tc::tmem_ld32(tO + lane_off + 32 * c, v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                    tc::tmem_st32(tO + lane_off + 32 * c, v);
                }
            }
            // pass 2: P = 2^(s * scale - m) (bf16) into the first 64 columns
            const float2 nm2 = make_float2(-msub, -msub);
            float2 sum2 = make_float2(0.f, 0.f), sum2b = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(tS + lane_off + 32 * c, v);
                tc::tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float2 x = tc::ffma2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), scale2, nm2);
                    float2 pe;
                    if (((e >> 1) & 3) < kPolyPairsOf4Sdpa) {
                        pe = tc::exp2_poly3_x2_ftz(x);
                    } else {
                        pe.x = ex2(x.x);
                        pe.y = ex2(x.y);
                    }
                    if (limit < 128) {
                        pe.x = (32 * c + e < limit) ? pe.x : 0.f;
                        pe.y = (32 * c + e + 1 < limit) ? pe.y : 0.f;
                    }
                    if ((e >> 1) & 1) sum2b = tc::fadd2_ftz(sum2b, pe);
                    else sum2 = tc::fadd2_ftz(sum2, pe);
                    pk[e >> 1] = tc::pack_bf16(pe.x, pe.y);
                }
                tc::tmem_st16(tS + lane_off + 16 * c, pk);
            }
            tc::tmem_st_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            const float sum = (sum2.x + sum2.y) + (sum2b.x + sum2b.y);
            l_run = l_run * alpha + sum;
            m_run = m_use;
        }
        // ------------------------------------------------------------ epilogue
        if (ok && warp_wait(pv_done, (nb - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag)) {
            fence_after_sync();
            const float inv = 1.f / l_run;
            __nv_bfloat16* orow = p.out + ((size_t)(b * p.Hq + h) * p.T + i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(tO + lane_off + 32 * c, v);
                tc::tmem_ld_wait();
                if (i < p.T) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 val;
                        val.x = tc::pack_bf16(__uint_as_float(v[8 * q4 + 0]) * inv, __uint_as_float(v[8 * q4 + 1]) * inv);
                        val.y = tc::pack_bf16(__uint_as_float(v[8 * q4 + 2]) * inv, __uint_as_float(v[8 * q4 + 3]) * inv);
                        val.z = tc::pack_bf16(__uint_as_float(v[8 * q4 + 4]) * inv, __uint_as_float(v[8 * q4 + 5]) * inv);
                        val.w = tc::pack_bf16(__uint_as_float(v[8 * q4 + 6]) * inv, __uint_as_float(v[8 * q4 + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q4) = val;
                    }
                }
            }
            if (i < p.T) p.lse[(size_t)(b * p.Hq + h) * p.tmax + i] = (m_run + log2f(l_run)) * kLn2;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tc::tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

// ============================================================================
// Weight sums
// ============================================================================
template <int D>
struct WsumCfg {
    static constexpr int QS = 2;                 // Q stages
    static constexpr int HALF = 128 * 128;
    static constexpr int TILE = 128 * D * 2;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_Q = OFF_K + TILE;
    static constexpr int OFF_ROW = OFF_Q + QS * TILE;     // part's rows x (float -lse2, int row)
    static constexpr int OFF_BAR = OFF_ROW + kRowsPerPart * 8;
    static constexpr int NBAR = 16;
    // at least ~80 KB so that no more than two CTAs (2 x 256 TMEM columns)
    // share an SM
    static constexpr int SMEM_MIN = 80 * 1024;
    static constexpr int SMEM_RAW = OFF_BAR + NBAR * 8 + 16 + 1024;
    static constexpr int SMEM = SMEM_RAW > SMEM_MIN ? SMEM_RAW : SMEM_MIN;
    static constexpr uint32_t IDESC = tc::idesc_bf16_f32(128, 128, false);
};

struct WsumParams {
    int B, Hq, Hkv, T, C, n, tmax;
    int G, rows_total, nparts, nbc, groups;
    float scale_log2;
    const float* lse;
    float* partials;   // [nparts][groups][C + tmax]
    WaitBound wb;
};

// Whether any row of tile [r0, r0 + 128) of the group's flattened rows
// (row = head * T + i) sees chunk token t0 or later (rows i >= t0 do).
__device__ __forceinline__ bool tile_visible(int r0, int rows_total, int T, int t0) {
    if (t0 <= 0) return true;
    const int last = min(r0 + 127, rows_total - 1);
    if (last / T > r0 / T) return true;  // the tile holds the end of a head
    return (last % T) >= t0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
wsum_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
               const __grid_constant__ CUtensorMap map_k, const WsumParams p) {
    using Cfg = WsumCfg<D>;
    constexpr int QS = Cfg::QS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* k_full = bars;
    uint64_t* q_full = k_full + 1;
    uint64_t* q_empty = q_full + QS;
    uint64_t* s_full = q_empty + QS;
    uint64_t* s_empty = s_full + 2;
    uint64_t* drain = s_empty + 2;
    uint64_t* rows_ready = drain + 1;  // 128 arrivals: the part's row table is in place
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* row_l2 = reinterpret_cast<float*>(smem + Cfg::OFF_ROW);                 // [kRowsPerPart]
    int* row_i = reinterpret_cast<int*>(smem + Cfg::OFF_ROW + kRowsPerPart * 4);    // [kRowsPerPart]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // unit = (key block, row part, group); cache key blocks (most rows) first
    const int u = blockIdx.x;
    const int bg = u % p.groups;
    const int part = (u / p.groups) % p.nparts;
    const int kb = u / (p.groups * p.nparts);
    const bool cache = kb < p.nbc;
    const int t0 = cache ? 0 : 128 * (kb - p.nbc);          // first chunk token of the block
    const int key_row = cache ? bg * p.C + 128 * kb : bg * p.T + t0;
    const int cand0 = cache ? 128 * kb : p.n + t0;          // candidate index of lane 0
    const int n_keys = cache ? min(128, p.n - 128 * kb) : min(128, p.T - t0);
    const int r_begin = part * kRowsPerPart;
    const int r_end = min(r_begin + kRowsPerPart, p.rows_total);
    const int n_tiles = r_end > r_begin ? (r_end - r_begin + 127) / 128 : 0;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int qhead0 = b * p.Hq + g * p.G;                  // first query head of the group

    if (threadIdx.x == 0) {
        mbar_init(k_full, 1);
        for (int s = 0; s < QS; ++s) {
            mbar_init(q_full + s, 1);
            mbar_init(q_empty + s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(s_full + s, 1);
            mbar_init(s_empty + s, 4);
        }
        mbar_init(rows_ready, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&map_q);
            int qcount[QS] = {};
            mbar_arrive_expect_tx(k_full, Cfg::TILE);
            const CUtensorMap* mk = cache ? &map_kc : &map_k;
            for (int hh = 0; hh < D / 64; ++hh)
                tc::tma_load_2d(smem + Cfg::OFF_K + hh * Cfg::HALF, mk, 64 * hh, key_row, k_full);
            int cnt = 0;
            for (int tt = 0; tt < n_tiles; ++tt) {
                const int r0 = r_begin + 128 * tt;
                if (!tile_visible(r0, p.rows_total, p.T, t0)) continue;
                const int qs = cnt % QS;
                if (!wait_bar(q_empty + qs, ((cnt / QS) & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag)) break;
                mbar_arrive_expect_tx(q_full + qs, Cfg::TILE);
                for (int hh = 0; hh < D / 64; ++hh)
                    tc::tma_load_2d(smem + Cfg::OFF_Q + qs * Cfg::TILE + hh * Cfg::HALF, &map_q, 64 * hh,
                                    qhead0 * p.T + r0, q_full + qs);
                ++qcount[qs];
                ++cnt;
            }
            wait_bar(k_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
            for (int s = 0; s < QS; ++s)
                if (qcount[s]) wait_bar(q_full + s, (qcount[s] - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
        }
    } else if (warp == 1) {
        bool ok = warp_wait(k_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
        const uint32_t sK = sbase + Cfg::OFF_K;
        int cnt = 0;
        for (int tt = 0; ok && tt < n_tiles; ++tt) {
            if (!tile_visible(r_begin + 128 * tt, p.rows_total, p.T, t0)) continue;
            const int qs = cnt % QS, sb = cnt & 1;
            ok = warp_wait(q_full + qs, (cnt / QS) & 1, p.wb, kDevTimeoutTmaWait, abort_flag) &&
                 warp_wait(s_empty + sb, ((cnt >> 1) & 1) ^ 1, p.wb, kDevTimeoutMmaWait, abort_flag);
            if (!ok) break;
            fence_after_sync();
            if (lane == 0) {
                const uint32_t sQ = sbase + Cfg::OFF_Q + qs * Cfg::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * Cfg::HALF + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + 128 * sb, desc_kmajor_sw128(sK + off), desc_kmajor_sw128(sQ + off),
                                    Cfg::IDESC, kk > 0);
                }
                tc::mma_commit(s_full + sb);
                tc::mma_commit(q_empty + qs);
            }
            __syncwarp();
            ++cnt;
        }
        if (lane == 0) tc::mma_commit(drain);
        __syncwarp();
        warp_wait(drain, 0, p.wb, kDevTimeoutMmaWait, abort_flag);
    } else {
        const int quad = warp & 3;
        const int tid = threadIdx.x - 64;      // 0..127: column helper index
        const int kr = quad * 32 + lane;       // key row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int t_key = cache ? -1 : t0 + kr;  // chunk token index of this key
        // the part's row table: minus the log2-domain LSE of each row (-inf
        // for rows outside the part) and its row index inside the chunk
        {
            constexpr int PER = kRowsPerPart / 128;
            float lv[PER];
            int iv[PER];
#pragma unroll
            for (int q = 0; q < PER; ++q) {  // all loads in flight at once
                const int fr = r_begin + tid + 128 * q;
                iv[q] = -1;
                lv[q] = INFINITY;
                if (fr < r_end) {
                    const int hh = fr / p.T;
                    iv[q] = fr - hh * p.T;
                    lv[q] = __ldg(p.lse + (size_t)(qhead0 + hh) * p.tmax + iv[q]);
                }
            }
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                row_l2[tid + 128 * q] = -lv[q] * kLog2e;
                row_i[tid + 128 * q] = iv[q];
            }
        }
        mbar_arrive(rows_ready);
        float acc = 0.f;
        int cnt = 0;
        bool ok = warp_wait(rows_ready, 0, p.wb, kDevTimeoutSlotWait, abort_flag);
        for (int tt = 0; ok && tt < n_tiles; ++tt) {
            const int r0 = r_begin + 128 * tt;
            if (!tile_visible(r0, p.rows_total, p.T, t0)) continue;
            const int sb = cnt & 1;
            ok = warp_wait(s_full + sb, (cnt >> 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
            if (!ok) break;
            fence_after_sync();
            float s[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(tmem + 128 * sb + lane_off + 32 * c, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(v[e]);
            }
            tc::tmem_ld_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty + sb);
            const float4* l2v = reinterpret_cast<const float4*>(row_l2 + 128 * tt);
            const int4* riv = reinterpret_cast<const int4*>(row_i + 128 * tt);
            // the causal mask matters only for chunk keys on tiles that hold a
            // row i < t0 + 127 (tiles inside one head starting at i >= t0+127
            // are fully visible)
            const int last = min(r0 + 127, r_end - 1);
            const bool masked = !cache && ((last / p.T != r0 / p.T) || (r0 % p.T) < t0 + 127);
            const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
            float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
#pragma unroll
            for (int c4 = 0; c4 < 32; ++c4) {
                const float4 L = l2v[c4];
                float2 w01 = tc::ffma2(make_float2(s[4 * c4], s[4 * c4 + 1]), scale2, make_float2(L.x, L.y));
                float2 w23 = tc::ffma2(make_float2(s[4 * c4 + 2], s[4 * c4 + 3]), scale2, make_float2(L.z, L.w));
                const int pair0 = 2 * c4, pair1 = 2 * c4 + 1;
                if ((pair0 & 7) < kPolyPairsOf8Wsum) {
                    w01 = tc::exp2_poly3_x2_ftz(w01);
                } else {
                    w01.x = ex2(w01.x);
                    w01.y = ex2(w01.y);
                }
                if ((pair1 & 7) < kPolyPairsOf8Wsum) {
                    w23 = tc::exp2_poly3_x2_ftz(w23);
                } else {
                    w23.x = ex2(w23.x);
                    w23.y = ex2(w23.y);
                }
                if (masked) {
                    const int4 I = riv[c4];
                    w01.x = (I.x >= t_key) ? w01.x : 0.f;
                    w01.y = (I.y >= t_key) ? w01.y : 0.f;
                    w23.x = (I.z >= t_key) ? w23.x : 0.f;
                    w23.y = (I.w >= t_key) ? w23.y : 0.f;
                }
                if (c4 & 1) {
                    a2 = tc::fadd2_ftz(a2, w01);
                    a3 = tc::fadd2_ftz(a3, w23);
                } else {
                    a0 = tc::fadd2_ftz(a0, w01);
                    a1 = tc::fadd2_ftz(a1, w23);
                }
            }
            const float tile_acc = ((a0.x + a0.y) + (a1.x + a1.y)) + ((a2.x + a2.y) + (a3.x + a3.y));
            acc += tile_acc;
            ++cnt;
        }
        if (ok && kr < n_keys)
            p.partials[((size_t)part * p.groups + bg) * (size_t)(p.C + p.tmax) + cand0 + kr] = acc;
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

// Device evaluation of the exp2 variants, for testing them against each other
// and against a high-precision reference.
__global__ void exp2_selftest_kernel(const float* x, float* y3, float* y4, float* ym, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    y3[i] = tc::exp2_poly3(x[i]);
    y4[i] = tc::exp2_poly4(x[i]);
    ym[i] = ex2(x[i]);
}

// ============================================================================
// host side
// ============================================================================
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D map over a [rows, d] bf16 matrix, boxes of 128 rows x 64 columns,
// 128-byte swizzle (the layout the UMMA descriptors above describe).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, int d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int nparts_for(int G, int T) { return (G * T + kRowsPerPart - 1) / kRowsPerPart; }

template <int D>
cudaError_t sdpa_launch(const StepArgs& a) {
    using Cfg = SdpaCfg<D>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(sdpa_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap mq, mkc, mvc, mk, mv;
    if (!make_map(&mq, a.q, (uint64_t)a.B * a.Hq * a.T, D) || !make_map(&mkc, a.Kc, (uint64_t)a.B * a.Hkv * a.C, D) ||
        !make_map(&mvc, a.Vc, (uint64_t)a.B * a.Hkv * a.C, D) || !make_map(&mk, a.k, (uint64_t)a.B * a.Hkv * a.T, D) ||
        !make_map(&mv, a.v, (uint64_t)a.B * a.Hkv * a.T, D))
        return cudaErrorInvalidValue;
    SdpaParams p;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.T = a.T;
    p.C = a.C;
    p.n = a.n;
    p.tmax = a.tmax;
    p.n_mblk = (a.T + 127) / 128;
    p.nbc = (a.n + 127) / 128;
    p.scale_log2 = kLog2e / sqrtf((float)D);
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.lse = a.lse;
    p.wb = a.wb;
    const int grid = p.n_mblk * a.B * a.Hq;
    sdpa_tc_kernel<D><<<grid, kThreads, Cfg::SMEM, a.stream>>>(mq, mkc, mvc, mk, mv, p);
    a.log->done("sdpa_tc_kernel", a.stream);
    return cudaGetLastError();
}

template <int D>
cudaError_t wsum_launch(const StepArgs& a) {
    using Cfg = WsumCfg<D>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(wsum_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int G = a.Hq / a.Hkv;
    const int groups = a.B * a.Hkv;
    const int nparts = nparts_for(G, a.T);
    if ((size_t)nparts * groups * (size_t)(a.C + a.tmax) > a.partial_elems) return cudaErrorInvalidValue;
    CUtensorMap mq, mkc, mk;
    if (!make_map(&mq, a.q, (uint64_t)a.B * a.Hq * a.T, D) || !make_map(&mkc, a.Kc, (uint64_t)a.B * a.Hkv * a.C, D) ||
        !make_map(&mk, a.k, (uint64_t)a.B * a.Hkv * a.T, D))
        return cudaErrorInvalidValue;
    WsumParams p;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.T = a.T;
    p.C = a.C;
    p.n = a.n;
    p.tmax = a.tmax;
    p.G = G;
    p.rows_total = G * a.T;
    p.nparts = nparts;
    p.nbc = (a.n + 127) / 128;
    p.groups = groups;
    p.scale_log2 = kLog2e / sqrtf((float)D);
    p.lse = a.lse;
    p.partials = a.partials;
    p.wb = a.wb;
    const int nbt = (a.T + 127) / 128;
    const int grid = (p.nbc + nbt) * nparts * groups;
    wsum_tc_kernel<D><<<grid, kThreads, Cfg::SMEM, a.stream>>>(mq, mkc, mk, p);
    a.log->done("wsum_tc_kernel", a.stream);
    return cudaGetLastError();
}

}  // namespace

bool tc_supported(int device, int d) {
    if (d != 64 && d != 128) return false;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess) return false;
    return major == 10 && minor == 0 && encode_fn() != nullptr;
}

size_t tc_partial_elems(int B, int Hq, int Hkv, int C, int tmax) {
    return (size_t)nparts_for(Hq / Hkv, tmax) * B * Hkv * (size_t)(C + tmax);
}

int tc_partial_count(int Hq, int Hkv, int T) { return nparts_for(Hq / Hkv, T); }

int tc_kernel_plan(int, int, int, int, int, int, int, const char** names, int max_names) {
    const char* plan[2] = {"sdpa_tc_kernel", "wsum_tc_kernel"};
    for (int i = 0; i < 2 && i < max_names; ++i) names[i] = plan[i];
    return 2;
}

cudaError_t tc_exp2_selftest(const float* x, float* y3, float* y4, float* ym, int n, cudaStream_t s) {
    exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, y3, y4, ym, n);
    return cudaGetLastError();
}

cudaError_t tc_sdpa(const StepArgs& a) { return a.d == 64 ? sdpa_launch<64>(a) : sdpa_launch<128>(a); }

cudaError_t tc_wsum(const StepArgs& a) { return a.d == 64 ? wsum_launch<64>(a) : wsum_launch<128>(a); }

}  // namespace h2o
