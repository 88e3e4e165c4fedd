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
// Both are warp-specialised: TMA loads and tcgen05.mma issue each have one
// elected lane of their own warp; 128-thread warpgroups own one TMEM lane
// (matrix row) per thread.
//
// SDPA: M = 128 query rows, N = 128 keys per block, K = d; two query tiles
//   (two heads of one KV group) per CTA, 11 warps: a loader (Q, and K / V
//   through a three-slot ring), one MMA-issuing warp per tile, and one softmax
//   warpgroup per tile. S = Q K^T lands in the tile's TMEM buffer; its softmax
//   warpgroup reads the row in one pass (S is then free for the next QK),
//   turns it into P (bf16, written to shared memory in the 128-byte-swizzled
//   K-major layout the next MMA reads, in two halves of 64 keys) and
//   O += P V accumulates in TMEM. The running maximum is only moved (and O
//   rescaled in TMEM) when it grows by more than 2^16, so most blocks skip the
//   rescale. One pair of exponentials in every four goes through a degree-3
//   polynomial on the FMA pipe, the rest through the MUFU unit.
// Weight sums: the transposed product S^T = K Q^T puts one KEY on each TMEM
//   lane (M = 128 keys) and 128 query rows on the columns, so each thread sums
//   its own key's weights across the columns in registers: the reduction over
//   queries needs no shuffles and no atomics. Query rows are split into parts
//   (per-CTA partials); the selection kernel adds the parts in a fixed order.
#include <cuda.h>

#include <algorithm>
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

// P may exceed 1 by up to 2^16 before the running maximum is moved: P is
// bf16 (same exponent range as fp32) and O and the row sum accumulate in fp32,
// so only overflow matters, and this keeps far from it.
constexpr float kRescaleThreshold = 16.f;  // log2 units
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

// ============================================================================
// SDPA
// ============================================================================
// One CTA per SM works on two query tiles at once: rows m0..m0+127 of query
// heads hA and hB = hA + 1 of the same KV group, so both see the same keys and
// every K/V block is loaded once for the pair. TMEM (512 columns) holds S and O
// (128 + d columns) per tile.
//
// Per key block j and tile X, the tile's softmax warpgroup reads the whole S
// row (128 fp32 values) into registers in one pass and releases S at once, so
// QK(j+1) runs on the tensor core while the exponentials of block j are
// computed. P goes to shared memory (bf16, 128-byte-swizzled, K-major) in two
// halves of 64 keys, each with its own full / consumed barriers: the PV MMA of
// the first half starts while the second half is computed, and the softmax of
// block j+1 only waits for the half of PV(j) whose buffer it overwrites.
// K and V blocks share a ring of three shared-memory slots, loaded in the
// order K0, K1, V0, K2, V1, ... so that each K block arrives a whole block
// before the QK that needs it.
// A group with an odd number of query heads leaves one single-tile CTA per
// (group, row tile).
template <int D>
struct SdpaCfg {
    static constexpr int HALF = 128 * 128;       // bytes of one 128-row x 64-col bf16 box
    static constexpr int TILE = 128 * D * 2;     // one 128-row x d tile
    static constexpr int PB = 2 * HALF;          // one P tile (128 rows x 128 keys, bf16), two halves
    static constexpr int RING = 3;               // K/V slots
    static constexpr int OFF_QA = 0;
    static constexpr int OFF_QB = TILE;
    static constexpr int OFF_RING = 2 * TILE;
    static constexpr int OFF_P = OFF_RING + RING * TILE;  // [2 tiles]
    static constexpr int OFF_BAR = OFF_P + 2 * PB;
    static constexpr int NBAR = 24;
    static constexpr int SMEM_RAW = OFF_BAR + NBAR * 8 + 16 + 1024;
    // more than half of an SM's shared memory, so one CTA (512 TMEM columns) per SM
    static constexpr int SMEM = SMEM_RAW > 120 * 1024 ? SMEM_RAW : 120 * 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    // warp 0 loads Q, K and V, warps 2..9 are the two softmax warpgroups,
    // warps 1 and 10 issue the MMAs of tiles A and B
    static constexpr int THREADS = 352;
    static constexpr uint32_t IDESC_QK = tc::idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(128, D, true);
};
static_assert(SdpaCfg<128>::SMEM_RAW <= 232448, "SDPA shared memory exceeds the per-CTA limit");

struct SdpaParams {
    int B, Hq, Hkv, T, C, n, tmax;
    int n_mblk;   // query-row tiles per head
    int nbc;      // cache key blocks = ceil(n / 128)
    int npairs;   // head pairs per KV group = ceil(G / 2)
    int rows_pad; // row stride of nlse2
    int nsplit;   // pieces the cache blocks of a unit are split into (1: none)
    int cb_per;   // cache blocks per piece
    int early;    // wait for the previous kernel only before the first cache
                  // block and before the epilogue (see sdpa_tc_kernel)
    float scale_log2;
    __nv_bfloat16* out;
    float* lse;
    float* nlse2;  // [groups][rows_pad]: -(log2-domain LSE) per flattened group row
    float* part_o;   // nsplit > 1: [nsplit][B*Hq*T][D] unnormalised partial outputs
    float* part_ml;  // nsplit > 1: [nsplit][B*Hq*T][2] their log2-domain maximum and sum
    WaitBound wb;
};

template <int D>
__global__ void __launch_bounds__(SdpaCfg<D>::THREADS, 1)
sdpa_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
               const __grid_constant__ CUtensorMap map_vc, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_v, const SdpaParams p) {
    using Cfg = SdpaCfg<D>;
    constexpr int RING = Cfg::RING;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* ring_full = bars + 1;            // [RING]
    uint64_t* ring_empty = ring_full + RING;   // [RING]
    uint64_t* s_full = ring_empty + RING;      // [2 tiles]
    uint64_t* s_free = s_full + 2;             // [2 tiles], 4 arrivals: S loaded into registers
    uint64_t* p_full = s_free + 2;             // [2 tiles][2 halves], 4 arrivals: P half in shared memory
    uint64_t* pv_done = p_full + 4;            // [2 tiles][2 halves]: PV of that half completed
    uint64_t* drain = pv_done + 4;             // [2 tiles]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // unit = (row tile, KV group, head pair); the last row tiles (most keys) first
    const int G = p.Hq / p.Hkv;
    const int per_mblk = p.B * p.Hkv * p.npairs;
    const int unit = blockIdx.x / p.nsplit, piece = blockIdx.x % p.nsplit;
    const int mblk = p.n_mblk - 1 - unit / per_mblk;
    const int rest = unit % per_mblk;
    const int bg = rest / p.npairs, pr = rest % p.npairs;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int hA = g * G + 2 * pr;
    const bool hasB = 2 * pr + 1 < G;
    const int m0 = mblk * 128;
    // this piece's key blocks: (in the last piece) the chunk blocks 0..mblk
    // first, then the cache blocks cb0 .. cb0 + ncb - 1; local block jj is
    // global block gblock(jj) (global numbering: cache blocks, then the
    // chunk's). The chunk's keys depend only on this step's inputs, so they go
    // first: in early mode they are attended to while the previous step's
    // eviction still runs.
    const bool last_piece = piece == p.nsplit - 1;
    const int cb0 = min(p.nbc, piece * p.cb_per);
    const int ncb = min(p.nbc, last_piece ? p.nbc : cb0 + p.cb_per) - cb0;
    const int nchk = last_piece ? mblk + 1 : 0;
    const int nb = nchk + ncb;
    auto gblock = [&](int jj) { return jj < nchk ? p.nbc + jj : cb0 + (jj - nchk); };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < RING; ++s) {
            mbar_init(ring_full + s, 1);
            mbar_init(ring_empty + s, hasB ? 2 : 1);  // released by each tile's MMA warp
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full + t, 1);
            mbar_init(s_free + t, 4);
            for (int h = 0; h < 2; ++h) {
                mbar_init(p_full + 2 * t + h, 4);
                mbar_init(pv_done + 2 * t + h, 1);
            }
        }
        mbar_init(drain, 1);
        mbar_init(drain + 1, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sbase = smem_u32(smem);
    // Early mode: the step's inputs (q, k, v) were complete before the
    // previous kernel on the stream started, so only the cache blocks (which
    // the previous step's eviction rewrites) and the writes of the epilogue
    // (buffers the previous step reads) wait for it; the loader and the
    // softmax warps each call griddep_wait() there. Otherwise every thread
    // waits here.
    if (!p.early) griddep_wait();  // inputs written, and the previous step's readers done
    griddep_launch_dependents();

    if (warp == 0) {
        // ----------------------------------------------------------- producer
        // Q of both tiles, then K0, K1, V0, K2, V1, ..., K(nb-1), V(nb-2), V(nb-1)
        // through the ring
        if (lane == 0) {
            tc::prefetch_tmap(&map_q);
            tc::prefetch_tmap(&map_kc);
            tc::prefetch_tmap(&map_vc);
            tc::prefetch_tmap(&map_k);
            tc::prefetch_tmap(&map_v);
            mbar_arrive_expect_tx(q_full, Cfg::TILE * (hasB ? 2 : 1));
            for (int hh = 0; hh < D / 64; ++hh) {
                tc::tma_load_2d(smem + Cfg::OFF_QA + hh * Cfg::HALF, &map_q, 64 * hh, (b * p.Hq + hA) * p.T + m0,
                                q_full);
                if (hasB)
                    tc::tma_load_2d(smem + Cfg::OFF_QB + hh * Cfg::HALF, &map_q, 64 * hh,
                                    (b * p.Hq + hA + 1) * p.T + m0, q_full);
            }
            int L = 0;
            bool waited = !p.early;
            auto load_kv = [&](bool isV, int jj) -> bool {
                const int j = gblock(jj);
                const int slot = L % RING;
                if (!wait_bar(ring_empty + slot, ((L / RING) & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag))
                    return false;
                const bool cache = j < p.nbc;
                if (cache && !waited) {
                    griddep_wait();  // the previous step's eviction has rewritten the cache
                    waited = true;
                }
                const int row = cache ? bg * p.C + 128 * j : bg * p.T + 128 * (j - p.nbc);
                const CUtensorMap* map = isV ? (cache ? &map_vc : &map_v) : (cache ? &map_kc : &map_k);
                mbar_arrive_expect_tx(ring_full + slot, Cfg::TILE);
                for (int hh = 0; hh < D / 64; ++hh)
                    tc::tma_load_2d(smem + Cfg::OFF_RING + slot * Cfg::TILE + hh * Cfg::HALF, map, 64 * hh, row,
                                    ring_full + slot);
                ++L;
                return true;
            };
            bool ok = load_kv(false, 0);
            for (int j = 0; ok && j < nb; ++j) {
                if (j + 1 < nb) ok = load_kv(false, j + 1);
                if (ok) ok = load_kv(true, j);
            }
            // every load issued here has landed before the CTA may exit
            wait_bar(q_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag);
            for (int s = 0; s < RING; ++s) {
                const int uses = L / RING + (s < L % RING ? 1 : 0);
                if (uses) wait_bar(ring_full + s, (uses - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
            }
        }
    } else if (warp == 1 || (warp == 10 && hasB)) {
        // ---------------------------------------------------------- MMA issuers
        // one warp per tile (warp 1: tile A, warp 10: tile B), so that the
        // waits and issue overhead of one tile overlap the other's; the
        // tensor core takes both streams. The whole warp runs the issue code
        // and elect.sync picks the lane that issues (measured 1.5 us faster
        // per launch than a lane-0 branch). Every descriptor is a base value
        // plus a constant offset (the start-address field is the byte
        // address / 16 in the low bits, and no address here reaches 2^18).
        const int X = warp == 1 ? 0 : 1;
        const uint32_t tS = tmem + 256 * X, tO = tmem + 256 * X + 128;
        const uint64_t dQ = desc_kmajor_sw128(sbase + (X ? Cfg::OFF_QB : Cfg::OFF_QA));
        const uint64_t dRingK = desc_kmajor_sw128(sbase + Cfg::OFF_RING);
        const uint64_t dRingV = desc_mnmajor_sw128(sbase + Cfg::OFF_RING, Cfg::HALF);
        const uint64_t dP = desc_kmajor_sw128(sbase + Cfg::OFF_P + X * Cfg::PB);
        auto issue_qk = [&](int slot) {
            const uint64_t dK = dRingK + (uint64_t)((slot * Cfg::TILE) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = ((kk >> 2) * Cfg::HALF + (kk & 3) * 32) >> 4;
                tc::mma_bf16_ss_warp(tS, dQ + off, dK + off, Cfg::IDESC_QK, kk > 0);
            }
        };
        // O += P[:, 64h .. 64h+63] V[64h .. 64h+63, :]
        auto issue_pv_half = [&](int slot, int h, bool first) {
            const uint64_t dV = dRingV + (uint64_t)((slot * Cfg::TILE) >> 4);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {  // 64 keys, 16 per instruction
                const int kk = 4 * h + k4;
                tc::mma_bf16_ss_warp(tO, dP + (uint64_t)((h * Cfg::HALF + k4 * 32) >> 4),
                                dV + (uint64_t)((kk * 16 * 128) >> 4), Cfg::IDESC_PV, (!first || k4 > 0) ? 1u : 0u);
            }
        };
        int L = 0;
        auto wait_ring = [&](int& slot) -> bool {
            slot = L % RING;
            const bool r = warp_wait(ring_full + slot, (L / RING) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
            ++L;
            return r;
        };
        int ks = 0;
        bool ok = warp_wait(q_full, 0, p.wb, kDevTimeoutTmaWait, abort_flag) && wait_ring(ks);
        if (ok) {
            {
                issue_qk(ks);
                tc::mma_commit_warp(s_full + X);
                tc::mma_commit_warp(ring_empty + ks);
            }
            __syncwarp();
        }
        for (int j = 0; ok && j < nb; ++j) {
            // QK(j + 1) as soon as the softmax has taken S(j) out of TMEM
            if (j + 1 < nb) {
                ok = wait_ring(ks) && warp_wait(s_free + X, j & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
                if (!ok) break;
                fence_after_sync();
                {
                    issue_qk(ks);
                    tc::mma_commit_warp(s_full + X);
                    tc::mma_commit_warp(ring_empty + ks);
                }
                __syncwarp();
            }
            // PV(j) half by half, as the softmax hands P over
            int vs = 0;
            if (!(ok = wait_ring(vs))) break;
            for (int h = 0; h < 2; ++h) {
                if (!(ok = warp_wait(p_full + 2 * X + h, j & 1, p.wb, kDevTimeoutMmaWait, abort_flag))) break;
                fence_after_sync();
                {
                    issue_pv_half(vs, h, j == 0 && h == 0);
                    tc::mma_commit_warp(pv_done + 2 * X + h);
                }
                __syncwarp();
            }
            if (!ok) break;
            tc::mma_commit_warp(ring_empty + vs);
            __syncwarp();
        }
        // all MMAs issued here complete before TMEM can be released
        tc::mma_commit_warp(drain + X);
        __syncwarp();
        warp_wait(drain + X, 0, p.wb, kDevTimeoutMmaWait, abort_flag);
    } else if (warp >= 2 && warp < 10 && (warp < 6 || hasB)) {
        // -------------------------------------------------------------- softmax
        const int X = warp < 6 ? 0 : 1;     // which tile
        const int h = hA + X;
        const uint32_t tS = tmem + 256 * X, tO = tmem + 256 * X + 128;
        uint8_t* prow_base = smem + Cfg::OFF_P + X * Cfg::PB;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // row inside the tile = TMEM lane
        const int i = m0 + r;            // query row inside the chunk
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        uint8_t* prow = prow_base + r * 128;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
            ok = warp_wait(s_full + X, j & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
            if (!ok) break;
            fence_after_sync();
            // the whole row of S in one pass; S is free for QK(j+1) right after
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld32(tS + lane_off + 32 * c, v[c]);
            tc::tmem_ld_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free + X);
            // visible columns of this row in block j: col < limit
            const int jg = gblock(j);
            const int limit = (jg < p.nbc) ? p.n - 128 * jg : min(i, p.T - 1) - 128 * (jg - p.nbc) + 1;
            if (limit < 128) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * c + e >= limit) v[c][e] = __float_as_uint(-INFINITY);
            }
            // row maximum of the raw scores (the scale is positive)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    mx0 = tc::max3(mx0, __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]));
                    mx1 = tc::max3(mx1, __uint_as_float(v[c][e + 2]), __uint_as_float(v[c][e + 3]));
                }
            // the running maximum only moves when it grows by more than 2^16
            const float m_new = fmaxf(m_run, fmaxf(mx0, mx1) * p.scale_log2);
            const bool resc = m_new > m_run + kRescaleThreshold;
            const float m_use = resc ? m_new : m_run;
            const float alpha = resc ? ex2(m_run - m_use) : 1.f;
            // P = 2^(s * scale - m) -> bf16 -> shared memory, one half of the
            // keys at a time
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
            const float2 nm2 = make_float2(-m_use, -m_use);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                // the half's buffer is free once PV(j-1) of the same half has
                // completed (after a give-up the stores are harmless: nothing
                // reads them)
                if (j > 0 && ok) ok = warp_wait(pv_done + 2 * X + hf, (j - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {  // 8 keys (16 bytes of P) at a time
                    const int c = 2 * hf + (cc >> 2);
                    const int e0 = 8 * (cc & 3);
                    uint32_t pk[4];
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        const float2 x = tc::ffma2(
                            make_float2(__uint_as_float(v[c][e0 + k]), __uint_as_float(v[c][e0 + k + 1])), sc2, nm2);
                        float2 pe;
                        if ((k >> 1) < kPolyPairsOf4Sdpa) {
                            pe = tc::exp2_poly3_x2_ftz(x);
                        } else {
                            pe.x = ex2(x.x);
                            pe.y = ex2(x.y);
                        }
                        if (limit < 128) {
                            const int col = 32 * c + e0 + k;
                            pe.x = col < limit ? pe.x : 0.f;
                            pe.y = col + 1 < limit ? pe.y : 0.f;
                        }
                        if ((k >> 1) & 1) acc1 = tc::fadd2_ftz(acc1, pe);
                        else acc0 = tc::fadd2_ftz(acc0, pe);
                        pk[k >> 1] = tc::pack_bf16(pe.x, pe.y);
                    }
                    *reinterpret_cast<uint4*>(prow + hf * Cfg::HALF + ((cc ^ (r & 7)) << 4)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
                if (hf == 0 && j > 0 && ok && __any_sync(0xffffffffu, resc)) {
                    // rescale O once PV(j-1) has completed (its last half implies
                    // both), before PV(j) accumulates into it
                    ok = warp_wait(pv_done + 2 * X + 1, (j - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag);
                    if (ok) {
                        fence_after_sync();
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            tc::tmem_ld32(tO + lane_off + 32 * c, o);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tc::tmem_st32(tO + lane_off + 32 * c, o);
                        }
                        tc::tmem_st_wait();
                    }
                }
                tc::fence_proxy_async_smem();
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full + 2 * X + hf);
            }
            if (!ok) break;
            l_run = l_run * alpha + ((acc0.x + acc0.y) + (acc1.x + acc1.y));
            m_run = m_use;
        }
        // ------------------------------------------------------------ epilogue
        if (p.early) griddep_wait();  // the previous step no longer reads out, lse, nlse2
        if (ok && p.nsplit > 1 && warp_wait(pv_done + 2 * X + 1, (nb - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag)) {
            // one piece of a split unit: the unnormalised output, its maximum
            // and its sum, for sdpa_combine_kernel
            fence_after_sync();
            const size_t row = (size_t)(b * p.Hq + h) * p.T + i;
            const size_t rows = (size_t)p.B * p.Hq * p.T;
            float* prow_o = p.part_o + ((size_t)piece * rows + row) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tO + lane_off + 32 * c, o);
                tc::tmem_ld_wait();
                if (i < p.T) {
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        *reinterpret_cast<float4*>(prow_o + 32 * c + 4 * q4) =
                            make_float4(__uint_as_float(o[4 * q4]), __uint_as_float(o[4 * q4 + 1]),
                                        __uint_as_float(o[4 * q4 + 2]), __uint_as_float(o[4 * q4 + 3]));
                }
            }
            if (i < p.T)
                *reinterpret_cast<float2*>(p.part_ml + ((size_t)piece * rows + row) * 2) = make_float2(m_run, l_run);
        } else if (ok && p.nsplit == 1 && warp_wait(pv_done + 2 * X + 1, (nb - 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag)) {
            fence_after_sync();
            const float inv = 1.f / l_run;
            __nv_bfloat16* orow = p.out + ((size_t)(b * p.Hq + h) * p.T + i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tO + lane_off + 32 * c, o);
                tc::tmem_ld_wait();
                if (i < p.T) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 val;
                        val.x = tc::pack_bf16(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
                        val.y = tc::pack_bf16(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
                        val.z = tc::pack_bf16(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
                        val.w = tc::pack_bf16(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q4) = val;
                    }
                }
            }
            if (i < p.T) {
                const float lse2 = m_run + log2f(l_run);
                p.lse[(size_t)(b * p.Hq + h) * p.tmax + i] = lse2 * kLn2;
                p.nlse2[(size_t)bg * p.rows_pad + (size_t)(h - g * G) * p.T + i] = -lse2;
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tc::tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

// Merges the pieces of split SDPA units, one warp per query row: with the
// pieces' log2-domain maxima m_s and sums l_s, M = max m_s,
// L = sum_s l_s 2^(m_s - M), O = sum_s 2^(m_s - M) O_s / L; writes O (bf16),
// the natural-log LSE and -log2 LSE per flattened group row.
template <int D>
__global__ void __launch_bounds__(256)
sdpa_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml, int nsplit, int Hq,
                    int Hkv, int T, int tmax, int rows_pad, int rows, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse, float* __restrict__ nlse2) {
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) / 32, lane = threadIdx.x % 32;
    if (row >= rows) return;  // warp-uniform
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part_ml[((size_t)s * rows + row) * 2]);
    float L = 0.f;
    float o[D / 32];
#pragma unroll
    for (int c = 0; c < D / 32; ++c) o[c] = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float2 ml = *reinterpret_cast<const float2*>(part_ml + ((size_t)s * rows + row) * 2);
        const float w = exp2f(ml.x - M);
        L = fmaf(ml.y, w, L);
        const float* po = part_o + ((size_t)s * rows + row) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) o[c] = fmaf(po[lane + 32 * c], w, o[c]);
    }
    const float inv = 1.f / L;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) out[(size_t)row * D + lane + 32 * c] = __float2bfloat16_rn(o[c] * inv);
    if (lane == 0) {
        const int bh = row / T, i = row % T, G = Hq / Hkv;
        const float lse2 = M + log2f(L);
        lse[(size_t)bh * tmax + i] = lse2 * kLn2;
        nlse2[(size_t)(bh / G) * rows_pad + (size_t)(bh % G) * T + i] = -lse2;
    }
}

// ============================================================================
// Weight sums
// ============================================================================
// Persistent, two CTAs per SM: each CTA walks a static list of units (KV
// group, 128-key block, 1024-row part) in decreasing amount of work. Per unit
// it holds the key block (the A operand, M = 128 keys) and the part's row
// table (-log2 LSE per query row, fetched with one bulk copy), and streams
// 128-row query tiles (the B operand, N = 128): S^T = K Q^T lands in one of
// two 128-column TMEM buffers, one key per lane. Two consumer warpgroups
// share every tile, one half of its columns each (four consumer warps per SM
// sub-partition over the two CTAs); each thread sums its key's weights
// exp2(s * scale - lse2) over its half's columns in registers, the halves
// meet in shared memory at the end of a unit and the first writes the key's
// partial; the selection kernel adds all partials of a key in a fixed order.
constexpr int kRowsPerUnit = 1024;
constexpr int kRowTile = 128;
constexpr int kTilesPerUnit = kRowsPerUnit / kRowTile;

template <int D>
struct WsumCfg {
    static constexpr int QS = 2;                   // Q tile stages
    static constexpr int HALF = 128 * 128;         // 128 rows x 64 cols box
    static constexpr int TILE = 128 * D * 2;
    static constexpr int OFF_K = 0;                           // key block
    static constexpr int OFF_Q = OFF_K + TILE;                // [QS] query tiles
    static constexpr int OFF_ROW = OFF_Q + QS * TILE;         // [2] row tables (-lse2)
    static constexpr int OFF_RED = OFF_ROW + 2 * kRowsPerUnit * 4;  // [2][128] second half's sums
    static constexpr int OFF_BAR = OFF_RED + 2 * 128 * 4;
    static constexpr int NBAR = 24;
    static constexpr int SMEM_RAW = OFF_BAR + NBAR * 8 + 16 + 1024;
    // at least ~80 KB so that no more than two CTAs (2 x 256 TMEM columns) share an SM
    static constexpr int SMEM = SMEM_RAW > 80 * 1024 ? SMEM_RAW : 80 * 1024;
    static constexpr int THREADS = 320;                       // producer, MMA, 8 consumer warps
    static constexpr uint32_t IDESC = tc::idesc_bf16_f32(128, kRowTile, false);
};

struct WsumParams {
    int B, Hq, Hkv, T, C, n, tmax;
    int G, rows_total, n_ru, nbc, nkb, groups, units, rows_pad;
    float scale_log2;
    const float* nlse2;   // [groups][rows_pad]: -(log2-domain LSE) per flattened row
    float* partials;      // [n_ru][groups][C + tmax]
    WaitBound wb;
};

struct WsumUnit {
    int bg, ru, kb;
    bool cache;
    int t0, key_row, cand0, n_keys, r_begin, r_end;
};

__device__ __forceinline__ WsumUnit wsum_unit(const WsumParams& p, int u) {
    WsumUnit w;
    w.bg = u % p.groups;
    w.ru = (u / p.groups) % p.n_ru;
    w.kb = u / (p.groups * p.n_ru);
    w.cache = w.kb < p.nbc;
    w.t0 = w.cache ? 0 : 128 * (w.kb - p.nbc);
    w.key_row = w.cache ? w.bg * p.C + 128 * w.kb : w.bg * p.T + w.t0;
    w.cand0 = w.cache ? 128 * w.kb : p.n + w.t0;
    w.n_keys = w.cache ? min(128, p.n - 128 * w.kb) : min(128, p.T - w.t0);
    w.r_begin = w.ru * kRowsPerUnit;
    w.r_end = min(w.r_begin + kRowsPerUnit, p.rows_total);
    return w;
}

// Whether any row of the 128-row tile starting at flattened row r0 (row =
// head * T + i) sees chunk token t0 or later (rows with i >= t0 do).
__device__ __forceinline__ bool wtile_visible(int r0, int r_end, int T, int t0) {
    if (r0 >= r_end) return false;
    if (t0 <= 0) return true;
    const int last = min(r0 + kRowTile - 1, r_end - 1);
    if (last / T > r0 / T) return true;  // the tile holds the end of a head
    return (last % T) >= t0;
}

// Persistent weight-sum kernel, two CTAs per SM (each 256 TMEM columns: two
// 128-column S^T buffers). A CTA walks units (KV group, 128-key block,
// 1024-row part) in decreasing amount of work; per unit it loads the key
// block once (the A operand, M = 128 keys) and the part's row table with one
// bulk copy, and streams 128-row query tiles (the B operand, N = 128).
template <int D>
__global__ void __launch_bounds__(WsumCfg<D>::THREADS, 2)
wsum_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
               const __grid_constant__ CUtensorMap map_k, const WsumParams p) {
    using Cfg = WsumCfg<D>;
    constexpr int QS = Cfg::QS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* k_full = bars;
    uint64_t* k_empty = bars + 1;
    uint64_t* r_full = bars + 2;        // [2]
    uint64_t* r_empty = bars + 4;       // [2], 4 consumer-warp arrivals
    uint64_t* q_full = bars + 6;        // [QS]
    uint64_t* q_empty = q_full + QS;    // [QS]
    uint64_t* s_full = q_empty + QS;    // [2]
    uint64_t* s_empty = s_full + 2;     // [2], 4 arrivals
    uint64_t* drain = s_empty + 2;
    uint64_t* red_full = drain + 1;     // [2], 4 arrivals: the second half's sums written
    uint64_t* red_empty = red_full + 2; // [2], 4 arrivals: read by the first half
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        mbar_init(k_full, 1);
        mbar_init(k_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(r_full + s, 1);
            mbar_init(r_empty + s, 8);
            mbar_init(s_full + s, 1);
            mbar_init(s_empty + s, 8);
            mbar_init(red_full + s, 4);
            mbar_init(red_empty + s, 4);
        }
        for (int s = 0; s < QS; ++s) {
            mbar_init(q_full + s, 1);
            mbar_init(q_empty + s, 1);
        }
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
    griddep_wait();  // the SDPA's LSE rows are written
    griddep_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::prefetch_tmap(&map_q);
            int uc = 0, qc = 0;
            int kn = 0, rn[2] = {0, 0}, qn[QS] = {};
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++uc) {
                const WsumUnit w = wsum_unit(p, u);
                const int st = uc & 1;
                // row table: -lse2 of the unit's rows (rounded up to 16 bytes)
                if (!(ok = wait_bar(r_empty + st, ((uc >> 1) & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag))) break;
                const uint32_t rbytes = (uint32_t)(((w.r_end - w.r_begin) + 3) & ~3) * 4u;
                mbar_arrive_expect_tx(r_full + st, rbytes);
                tc::bulk_load(smem + Cfg::OFF_ROW + st * kRowsPerUnit * 4,
                              p.nlse2 + (size_t)w.bg * p.rows_pad + w.r_begin, rbytes, r_full + st);
                ++rn[st];
                // key block, once the previous unit's MMAs are done with it
                if (!(ok = wait_bar(k_empty, (uc & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag))) break;
                mbar_arrive_expect_tx(k_full, Cfg::TILE);
                const CUtensorMap* mk = w.cache ? &map_kc : &map_k;
                for (int hh = 0; hh < D / 64; ++hh)
                    tc::tma_load_2d(smem + Cfg::OFF_K + hh * Cfg::HALF, mk, 64 * hh, w.key_row, k_full);
                ++kn;
                // query tiles
                const int b = w.bg / p.Hkv, g = w.bg % p.Hkv;
                const int qrow0 = (b * p.Hq + g * p.G) * p.T;
                for (int tt = 0; tt < kTilesPerUnit; ++tt) {
                    const int r0 = w.r_begin + kRowTile * tt;
                    if (!wtile_visible(r0, w.r_end, p.T, w.t0)) continue;
                    const int qs = qc % QS;
                    if (!(ok = wait_bar(q_empty + qs, ((qc / QS) & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag)))
                        break;
                    mbar_arrive_expect_tx(q_full + qs, Cfg::TILE);
                    for (int hh = 0; hh < D / 64; ++hh)
                        tc::tma_load_2d(smem + Cfg::OFF_Q + qs * Cfg::TILE + hh * Cfg::HALF, &map_q, 64 * hh,
                                        qrow0 + r0, q_full + qs);
                    ++qn[qs];
                    ++qc;
                }
            }
            // every load issued here has landed before the CTA may exit
            if (kn) wait_bar(k_full, (kn - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
            for (int s = 0; s < 2; ++s)
                if (rn[s]) wait_bar(r_full + s, (rn[s] - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
            for (int s = 0; s < QS; ++s)
                if (qn[s]) wait_bar(q_full + s, (qn[s] - 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag);
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------- MMA issuer
        int uc = 0, qc = 0, tc_ = 0;
        bool ok = true;
        // descriptors: a base value plus constant offsets (start address >> 4)
        const uint64_t dK = desc_kmajor_sw128(sbase + Cfg::OFF_K);
        const uint64_t dQ0 = desc_kmajor_sw128(sbase + Cfg::OFF_Q);
        for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++uc) {
            const WsumUnit w = wsum_unit(p, u);
            if (!(ok = warp_wait(k_full, uc & 1, p.wb, kDevTimeoutTmaWait, abort_flag))) break;
            for (int tt = 0; tt < kTilesPerUnit; ++tt) {
                if (!wtile_visible(w.r_begin + kRowTile * tt, w.r_end, p.T, w.t0)) continue;
                const int qs = qc % QS, sb = tc_ & 1;
                ok = warp_wait(q_full + qs, (qc / QS) & 1, p.wb, kDevTimeoutTmaWait, abort_flag) &&
                     warp_wait(s_empty + sb, ((tc_ >> 1) & 1) ^ 1, p.wb, kDevTimeoutMmaWait, abort_flag);
                if (!ok) break;
                fence_after_sync();
                if (lane == 0) {
                    const uint64_t dQ = dQ0 + (uint64_t)((qs * Cfg::TILE) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = (uint64_t)(((kk >> 2) * Cfg::HALF + (kk & 3) * 32) >> 4);
                        tc::mma_bf16_ss(tmem + 128 * sb, dK + off, dQ + off, Cfg::IDESC, kk > 0);
                    }
                    tc::mma_commit(s_full + sb);
                    tc::mma_commit(q_empty + qs);
                }
                __syncwarp();
                ++qc;
                ++tc_;
            }
            if (!ok) break;
            if (lane == 0) tc::mma_commit(k_empty);  // after the unit's last MMA
            __syncwarp();
        }
        if (lane == 0) tc::mma_commit(drain);
        __syncwarp();
        warp_wait(drain, 0, p.wb, kDevTimeoutMmaWait, abort_flag);
    } else {
        // ------------------------------------------------------------ consumers
        const int quad = warp & 3;
        const int kr = quad * 32 + lane;         // key row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int half = (warp - 2) >> 2;        // columns 64 * half .. 64 * half + 63 of every tile
        const int cb = 64 * half;
        float* red = reinterpret_cast<float*>(smem + Cfg::OFF_RED);
        int uc = 0, tc_ = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++uc) {
            const WsumUnit w = wsum_unit(p, u);
            const int st = uc & 1;
            if (!(ok = warp_wait(r_full + st, (uc >> 1) & 1, p.wb, kDevTimeoutTmaWait, abort_flag))) break;
            const float* rowt = reinterpret_cast<const float*>(smem + Cfg::OFF_ROW + st * kRowsPerUnit * 4);
            const int t_key = w.cache ? -1 : w.t0 + kr;  // chunk token index of this key
            float acc = 0.f;
            for (int tt = 0; tt < kTilesPerUnit; ++tt) {
                const int r0 = w.r_begin + kRowTile * tt;
                if (!wtile_visible(r0, w.r_end, p.T, w.t0)) continue;
                const int sb = tc_ & 1;
                const int tcur = tc_++;
                if (!(ok = warp_wait(s_full + sb, (tcur >> 1) & 1, p.wb, kDevTimeoutMmaWait, abort_flag))) break;
                fence_after_sync();
                // this half's 64 columns of the tile in two chunks of 32: the
                // second chunk's TMEM load is in flight while the first is
                // summed, and the buffer is released as soon as it has landed
                const uint32_t tS = tmem + 128 * sb + lane_off + cb;
                const int ncols = min(kRowTile, w.r_end - r0);  // valid rows in the tile
                const int last = min(r0 + kRowTile - 1, w.r_end - 1);
                const bool causal = !w.cache && ((last / p.T != r0 / p.T) || (r0 % p.T) < w.t0 + 127);
                const bool fast = ncols == kRowTile && !causal;
                const float* rt = rowt + kRowTile * tt;
                float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
                auto sum_chunk = [&](const uint32_t(&v)[32], int c0) {
                    if (fast) {
                        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 Lr = *reinterpret_cast<const float4*>(rt + c0 + 4 * q4);
                            float2 w01 = tc::ffma2(make_float2(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1])),
                                                   sc2, make_float2(Lr.x, Lr.y));
                            float2 w23 = tc::ffma2(make_float2(__uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3])),
                                                   sc2, make_float2(Lr.z, Lr.w));
                            if (q4 < kPolyPairsOf8Wsum) {
                                w01 = tc::exp2_poly3_x2_ftz(w01);
                                w23 = tc::exp2_poly3_x2_ftz(w23);
                            } else {
                                w01 = make_float2(ex2(w01.x), ex2(w01.y));
                                w23 = make_float2(ex2(w23.x), ex2(w23.y));
                            }
                            // flush-to-zero adds: the polynomial exp2 leaves values
                            // below 2^-126 as subnormals, which must count as 0
                            a01 = tc::fadd2_ftz(a01, w01);
                            a23 = tc::fadd2_ftz(a23, w23);
                        }
                    } else {
                        // rows past the part's end, or a causal chunk key: row i
                        // of column c (i advances with c and wraps at the head end)
                        int i = (r0 + c0) % p.T;
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int c = c0 + e;
                            const float wv = ex2(fmaf(__uint_as_float(v[e]), p.scale_log2, rt[c]));
                            const bool vis = (c < ncols) && (i >= t_key);
                            a01.x = tc::fadd_ftz(a01.x, vis ? wv : 0.f);
                            if (++i == p.T) i = 0;
                        }
                    }
                };
                uint32_t va[32], vb[32];
                tc::tmem_ld32(tS, va);
                tc::tmem_ld_wait();
                tc::reg_fence(va);
                tc::tmem_ld32(tS + 32, vb);
                sum_chunk(va, cb);
                tc::tmem_ld_wait();
                tc::reg_fence(vb);
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_empty + sb);
                sum_chunk(vb, cb + 32);
                acc += (a01.x + a01.y) + (a23.x + a23.y);
            }
            if (!ok) break;
            // the two halves' sums of a key meet in shared memory; the first
            // half adds them (first + second, a fixed order) and writes the
            // unit's partial
            float* rs = red + st * 128;
            if (half == 1) {
                if (!(ok = warp_wait(red_empty + st, ((uc >> 1) & 1) ^ 1, p.wb, kDevTimeoutSlotWait, abort_flag)))
                    break;
                rs[kr] = acc;
                __syncwarp();
                if (lane == 0) mbar_arrive(red_full + st);
            } else {
                if (!(ok = warp_wait(red_full + st, (uc >> 1) & 1, p.wb, kDevTimeoutSlotWait, abort_flag))) break;
                const float tot = acc + rs[kr];
                __syncwarp();
                if (lane == 0) mbar_arrive(red_empty + st);
                if (kr < w.n_keys)
                    p.partials[((size_t)w.ru * p.groups + w.bg) * (size_t)(p.C + p.tmax) + w.cand0 + kr] = tot;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(r_empty + st);
        }
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

// 2-D map over a [rows, d] bf16 matrix, boxes of box_rows rows x 64 columns,
// 128-byte swizzle (the layout the UMMA descriptors above describe).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int nparts_for(int G, int T) { return (G * T + kRowsPerUnit - 1) / kRowsPerUnit; }

// Pieces the cache blocks of each SDPA unit are split into: only when the
// units (query tiles x KV groups x head pairs) fill less than half of the SMs
// and the cache is long enough that each piece keeps at least two blocks.
int sdpa_split_count(int B, int Hq, int Hkv, int T, int n, int num_sms, int* cb_per = nullptr) {
    const int units = ((T + 127) / 128) * B * Hkv * ((Hq / Hkv + 1) / 2);
    const int nbc = (n + 127) / 128;
    int ns = 1;
    if (units * 2 <= num_sms && nbc >= 4) ns = std::max(1, std::min({num_sms / units, nbc / 2, 8}));
    // equal pieces of cb cache blocks (the last one takes the rest and the
    // chunk's blocks): every piece has at least one block
    const int cb = (nbc + ns - 1) / ns;
    if (ns > 1) ns = (nbc + cb - 1) / cb;
    if (cb_per) *cb_per = cb;
    return ns;
}

template <int D>
cudaError_t sdpa_launch(const StepArgs& a) {
    using Cfg = SdpaCfg<D>;
    if (cudaError_t e = ensure_smem_limit(sdpa_tc_kernel<D>, Cfg::SMEM); e != cudaSuccess) return e;
    CUtensorMap mq, mkc, mvc, mk, mv;
    if (!make_map(&mq, a.q, (uint64_t)a.B * a.Hq * a.T, D, 128) ||
        !make_map(&mkc, a.Kc, (uint64_t)a.B * a.Hkv * a.C, D, 128) ||
        !make_map(&mvc, a.Vc, (uint64_t)a.B * a.Hkv * a.C, D, 128) ||
        !make_map(&mk, a.k, (uint64_t)a.B * a.Hkv * a.T, D, 128) ||
        !make_map(&mv, a.v, (uint64_t)a.B * a.Hkv * a.T, D, 128))
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
    p.npairs = (a.Hq / a.Hkv + 1) / 2;
    p.rows_pad = a.rows_pad;
    p.scale_log2 = kLog2e / sqrtf((float)D);
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.lse = a.lse;
    p.nlse2 = a.nlse2;
    p.wb = a.wb;
    p.early = a.early;
    p.nsplit = sdpa_split_count(a.B, a.Hq, a.Hkv, a.T, a.n, a.num_sms, &p.cb_per);
    const size_t rows = (size_t)a.B * a.Hq * a.T;
    p.part_o = a.sdpa_part;
    p.part_ml = a.sdpa_part ? a.sdpa_part + (size_t)p.nsplit * rows * D : nullptr;
    if (p.nsplit > 1 && (!a.sdpa_part || a.sdpa_part_elems < (size_t)p.nsplit * rows * (D + 2)))
        return cudaErrorInvalidValue;
    const int grid = p.n_mblk * a.B * a.Hkv * p.npairs * p.nsplit;
    // early mode: launched as a programmatic dependent of the previous step's
    // selection, so its CTAs start on the free SMs while that still runs
    cudaError_t e = a.early ? launch_ex(true, sdpa_tc_kernel<D>, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM, a.stream,
                                        mq, mkc, mvc, mk, mv, p)
                            : launch_pdl(sdpa_tc_kernel<D>, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM, a.stream,
                                         mq, mkc, mvc, mk, mv, p);
    if (e != cudaSuccess) return e;
    a.log->done("sdpa_tc_kernel", a.stream);
    if (p.nsplit > 1) {
        const int blocks = (int)((rows * 32 + 255) / 256);
        sdpa_combine_kernel<D><<<blocks, 256, 0, a.stream>>>(p.part_o, p.part_ml, p.nsplit, a.Hq, a.Hkv, a.T, a.tmax,
                                                             a.rows_pad, (int)rows, p.out, p.lse, p.nlse2);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        a.log->done("sdpa_combine_kernel", a.stream);
    }
    return cudaGetLastError();
}

template <int D>
cudaError_t wsum_launch(const StepArgs& a) {
    using Cfg = WsumCfg<D>;
    if (cudaError_t e = ensure_smem_limit(wsum_tc_kernel<D>, Cfg::SMEM); e != cudaSuccess) return e;
    const int G = a.Hq / a.Hkv;
    const int groups = a.B * a.Hkv;
    const int n_ru = (G * a.T + kRowsPerUnit - 1) / kRowsPerUnit;
    if ((size_t)n_ru * groups * (size_t)(a.C + a.tmax) > a.partial_elems) return cudaErrorInvalidValue;
    CUtensorMap mq, mkc, mk;
    if (!make_map(&mq, a.q, (uint64_t)a.B * a.Hq * a.T, D, kRowTile) ||
        !make_map(&mkc, a.Kc, (uint64_t)a.B * a.Hkv * a.C, D, 128) ||
        !make_map(&mk, a.k, (uint64_t)a.B * a.Hkv * a.T, D, 128))
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
    p.n_ru = n_ru;
    p.nbc = (a.n + 127) / 128;
    p.nkb = p.nbc + (a.T + 127) / 128;
    p.groups = groups;
    p.units = p.nkb * n_ru * groups;
    p.rows_pad = a.rows_pad;
    p.scale_log2 = kLog2e / sqrtf((float)D);
    p.nlse2 = a.nlse2;
    p.partials = a.partials;
    p.wb = a.wb;
    const int grid = min(p.units, 2 * a.num_sms);
    cudaError_t e = launch_pdl(wsum_tc_kernel<D>, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM, a.stream, mq, mkc, mk, p);
    if (e != cudaSuccess) return e;
    a.log->done("wsum_tc_kernel", a.stream);
    return cudaGetLastError();
}

}  // namespace

bool tc_make_map(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_rows) {
    return make_map(m, base, rows, d, box_rows);
}

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

int tc_rows_pad(int Hq, int Hkv, int tmax) {
    const int rows = (Hq / Hkv) * tmax;
    return (rows + kRowsPerUnit - 1) / kRowsPerUnit * kRowsPerUnit;
}

int tc_partial_count(int Hq, int Hkv, int T) { return nparts_for(Hq / Hkv, T); }

int tc_kernel_plan(int B, int Hq, int Hkv, int, int, int T, int n, int num_sms, const char** names, int max_names) {
    const bool split = sdpa_split_count(B, Hq, Hkv, T, n, num_sms) > 1;
    const char* plan[3] = {"sdpa_tc_kernel", split ? "sdpa_combine_kernel" : "wsum_tc_kernel", "wsum_tc_kernel"};
    const int k = split ? 3 : 2;
    for (int i = 0; i < k && i < max_names; ++i) names[i] = plan[i];
    return k;
}

size_t tc_sdpa_part_elems(int B, int Hq, int Hkv, int d, int T, int n, int num_sms) {
    const int ns = sdpa_split_count(B, Hq, Hkv, T, n, num_sms);
    return ns > 1 ? (size_t)ns * B * Hq * T * (d + 2) : 0;
}

cudaError_t tc_exp2_selftest(const float* x, float* y3, float* y4, float* ym, int n, cudaStream_t s) {
    exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, y3, y4, ym, n);
    return cudaGetLastError();
}

cudaError_t tc_sdpa(const StepArgs& a) { return a.d == 64 ? sdpa_launch<64>(a) : sdpa_launch<128>(a); }

cudaError_t tc_wsum(const StepArgs& a) { return a.d == 64 ? wsum_launch<64>(a) : wsum_launch<128>(a); }

}  // namespace h2o
