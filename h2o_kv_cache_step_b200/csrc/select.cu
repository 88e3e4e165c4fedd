// select.cu -- H2O eviction: which C of the (n valid cache slots + T chunk
// tokens) candidates survive, where the surviving chunk tokens go, and the
// copy of their keys and values into the cache.
//
// "Learning how to Forget", paper page, section "Improvements to
// Heavy-Hitter Oracle (H2O)": new content overwrites the slots whose H2O
// score is smallest. Readings taken here: candidates are the cache slots and
// the chunk tokens together (a chunk token can be dropped at once); the C
// largest scores survive, equal scores resolved toward the larger (more
// recent) position; kept cache entries do not move and the kept chunk
// tokens, in position order, take the free slots in ascending slot order.
//
// Selection runs one CTA per (sequence, KV head): an MSB-first radix select
// over 64-bit keys (order-preserving score bits : position) finds the C-th
// largest key; block-wide scans then build the free-slot list and the token
// to slot map, and the same CTA copies the kept chunk tokens' key and value
// rows into their slots. Once the cache is full few chunk tokens outlive
// their own step (a few dozen of 1024 on the bench's workloads), so the copy
// is small, and keeping it here leaves every other SM to the next step's
// attention, which starts on its chunk-only key blocks while this kernel runs.
// (scatter_kernel, a wide grid of the same copies, serves insert-always.)
#include "kernels.h"

namespace h2o {
namespace {

constexpr int kSelThreads = 1024;

// fp32 score -> unsigned int whose unsigned order is the float order (-0 and
// +0 compare equal, as floats do).
__device__ __forceinline__ uint32_t ordered_bits(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Eviction ranking value of a candidate: its H2O score (sum policy), or the
// score over its age t - t_j with t = P + T the token count after the step
// (normalized policy; "Learning how to Forget", paper page, section
// "Improvements to Heavy-Hitter Oracle (H2O)"). fp32, division rounded to
// nearest, so that a host replay in fp32 ranks identically.
__device__ __forceinline__ float rank_value(float score, int32_t pos, int policy, long long t_after) {
    return policy == 1 ? __fdiv_rn(score, (float)(t_after - (long long)pos)) : score;
}

__device__ __forceinline__ uint64_t cand_key(const float* cs, const int32_t* cp, int c, int policy,
                                             long long t_after) {
    return ((uint64_t)ordered_bits(rank_value(cs[c], cp[c], policy, t_after)) << 32) | (uint32_t)cp[c];
}

// Candidate keys are staged in shared memory when they fit (the radix passes
// then read them from there), otherwise rebuilt from global memory per pass.
// The kept flags and the free-slot list always live in shared memory.
constexpr int kSelectSmemLimit = 220 * 1024;

// Exclusive prefix sum of one value per thread over the block; *total gets
// the sum. Uses `scratch` (>= 33 values of shared memory).
template <typename V>
__device__ V block_exclusive_scan(V v, V* scratch, V* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    V x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const V y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        V w = lane < nwarps ? scratch[lane] : V(0);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const V y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < nwarps) scratch[lane] = w;  // inclusive warp totals
        if (lane == 31) scratch[32] = w;
    }
    __syncthreads();
    const V base = warp > 0 ? scratch[warp - 1] : V(0);
    *total = scratch[32];
    const V r = base + x - v;
    __syncthreads();
    return r;
}

constexpr int kCandPerThread = 4;  // candidates a thread loads per round
constexpr int kFewEvictions = 8;   // up to this many evictions: repeated block minima
constexpr int kPartBatch = 4;      // weight-sum partials loaded per batch

// One CTA per (sequence, KV head). Shared memory: the 64-bit candidate keys
// (when SMEM_KEYS), the kept flags, the free-slot list and the kept chunk
// tokens in position order.
template <bool SMEM_KEYS>
__global__ void __launch_bounds__(kSelThreads)
select_kernel(float* __restrict__ cand_score, int32_t* __restrict__ cand_pos,
              uint8_t* __restrict__ cand_kept, int32_t* __restrict__ token_slot,
              float* __restrict__ scores, int32_t* __restrict__ pos,
              const float* __restrict__ partials, int nparts, int C, int T, int n, int tmax, long long P,
              int policy, const uint4* __restrict__ kin, const uint4* __restrict__ vin, uint4* __restrict__ Kc,
              uint4* __restrict__ Vc, int row_vecs) {
    __shared__ unsigned int hist[256];
    __shared__ unsigned long long scan_scratch[33];
    __shared__ unsigned long long red_min[32], red_max[32];
    __shared__ unsigned long long sh_prefix, sh_prefix_min;
    __shared__ int sh_hi, sh_krem, sh_done;
    extern __shared__ __align__(16) unsigned char dyn[];

    // the next kernel may start now: it waits for this one before it reads the
    // cache or writes anything this kernel reads
    griddep_launch_dependents();
    griddep_wait();  // the weight-sum partials are written
    const size_t bg = blockIdx.x;
    const int m = n + T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* cs = cand_score + bg * (size_t)(C + tmax);
    int32_t* cp = cand_pos + bg * (size_t)(C + tmax);
    uint8_t* kept_g = cand_kept + bg * (size_t)(C + tmax);
    int32_t* ts = token_slot + bg * (size_t)tmax;
    float* sc = scores + bg * (size_t)C;
    int32_t* ps = pos + bg * (size_t)C;
    // shared layout: [keys m x 8 B (SMEM_KEYS)] [kept m B] [free list C x 4 B]
    // [kept tokens T x 4 B]
    unsigned long long* skeys = reinterpret_cast<unsigned long long*>(dyn);
    uint8_t* skept = dyn + (SMEM_KEYS ? (size_t)m * 8 : 0);
    int32_t* sfree = reinterpret_cast<int32_t*>(skept + (((size_t)m + 15) & ~(size_t)15));
    int32_t* stok = sfree + C;

    // ---- 0. candidate scores (old score + weight-sum partials in a fixed
    // part order), positions and keys; every load of a round is issued
    // before any is used. Also the smallest and largest key.
    unsigned long long kmin = ~0ull, kmax = 0ull;
    for (int c0 = threadIdx.x; c0 < m; c0 += kCandPerThread * blockDim.x) {
        float sv[kCandPerThread];
        int32_t pv[kCandPerThread];
#pragma unroll
        for (int u = 0; u < kCandPerThread; ++u) {
            const int c = c0 + u * blockDim.x;
            sv[u] = 0.f;
            pv[u] = 0;
            if (c < m) {
                if (nparts > 0) {
                    sv[u] = c < n ? sc[c] : 0.f;
                    pv[u] = c < n ? ps[c] : (int32_t)(P + (c - n));
                } else {
                    sv[u] = cs[c];
                    pv[u] = cp[c];
                }
            }
        }
        if (nparts > 0) {
            const size_t pstride = (size_t)gridDim.x * (C + tmax);
            const float* pb = partials + bg * (size_t)(C + tmax);
            for (int q0 = 0; q0 < nparts; q0 += kPartBatch) {
                float t[kPartBatch][kCandPerThread];
#pragma unroll
                for (int qq = 0; qq < kPartBatch; ++qq)
#pragma unroll
                    for (int u = 0; u < kCandPerThread; ++u) {
                        const int c = c0 + u * blockDim.x;
                        t[qq][u] = (q0 + qq < nparts && c < m) ? pb[(size_t)(q0 + qq) * pstride + c] : 0.f;
                    }
#pragma unroll
                for (int qq = 0; qq < kPartBatch; ++qq)
#pragma unroll
                    for (int u = 0; u < kCandPerThread; ++u) sv[u] += t[qq][u];  // + 0 for absent parts is exact
            }
        }
#pragma unroll
        for (int u = 0; u < kCandPerThread; ++u) {
            const int c = c0 + u * blockDim.x;
            if (c >= m) continue;
            if (nparts > 0) {
                cs[c] = sv[u];
                cp[c] = pv[u];
            }
            // a cache slot's stored score becomes its new score now; if the
            // slot is evicted, placement (phase 4) overwrites it after the
            // barriers in between (with a chunk token's score, or 0)
            if (c < n) sc[c] = sv[u];
            const unsigned long long key =
                ((uint64_t)ordered_bits(rank_value(sv[u], pv[u], policy, P + T)) << 32) | (uint32_t)pv[u];
            if (SMEM_KEYS) skeys[c] = key;
            kmin = key < kmin ? key : kmin;
            kmax = key > kmax ? key : kmax;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, off);
        const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, off);
        kmin = a < kmin ? a : kmin;
        kmax = b > kmax ? b : kmax;
    }
    if (lane == 0) {
        red_min[warp] = kmin;
        red_max[warp] = kmax;
    }
    __syncthreads();
    if (warp == 0) {
        const int nwarps = (int)(blockDim.x >> 5);
        kmin = lane < nwarps ? red_min[lane] : ~0ull;
        kmax = lane < nwarps ? red_max[lane] : 0ull;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, off);
            const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, off);
            kmin = a < kmin ? a : kmin;
            kmax = b > kmax ? b : kmax;
        }
    }
    if (threadIdx.x == 0) {
        // the leading bits every key shares need no radix pass
        const int common = (m > 0 && kmin != kmax) ? __clzll((long long)(kmin ^ kmax)) : 64;
        sh_hi = 64 - common;
        sh_prefix = sh_hi >= 64 ? 0ull : (kmax >> sh_hi);
        sh_krem = C;
        sh_done = (m <= C) || sh_hi == 0;
        sh_prefix_min = kmin;
    }
    __syncthreads();
    auto key_of = [&](int c) -> uint64_t {
        return SMEM_KEYS ? (uint64_t)skeys[c] : cand_key(cs, cp, c, policy, P + T);
    };

    // few evictions (short chunks): the threshold is the k-th smallest key,
    // found by k - 1 block minima above the smallest one; no radix pass
    if (m > C && m - C <= kFewEvictions) {
        unsigned long long thr = sh_prefix_min;
        for (int it = 1; it < m - C; ++it) {
            unsigned long long lm = ~0ull;
            for (int c = threadIdx.x; c < m; c += blockDim.x) {
                const unsigned long long key = key_of(c);
                if (key > thr && key < lm) lm = key;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const unsigned long long o = __shfl_xor_sync(0xffffffffu, lm, off);
                lm = o < lm ? o : lm;
            }
            if (lane == 0) red_min[warp] = lm;
            __syncthreads();
            if (warp == 0) {
                lm = lane < (int)(blockDim.x >> 5) ? red_min[lane] : ~0ull;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const unsigned long long o = __shfl_xor_sync(0xffffffffu, lm, off);
                    lm = o < lm ? o : lm;
                }
                if (lane == 0) sh_prefix_min = lm;
            }
            __syncthreads();
            thr = sh_prefix_min;
        }
        if (threadIdx.x == 0) {  // kept iff key > thr
            sh_hi = 0;
            sh_prefix = thr + 1ull;
            sh_done = 1;
        }
        __syncthreads();
    }

    // ---- 1. threshold: the C-th largest key, MSB-first radix select over the
    // bits below the shared prefix, 8 bits a pass; it stops as soon as the
    // remaining keys fill one bin exactly
    while (!sh_done) {
        const int hi = sh_hi, lo = hi > 8 ? hi - 8 : 0;
        const unsigned long long prefix = sh_prefix;
        const unsigned long long dmask = (1ull << (hi - lo)) - 1ull;
        for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0u;
        __syncthreads();
        for (int c = threadIdx.x; c < m; c += blockDim.x) {
            const uint64_t key = key_of(c);
            if ((hi >= 64) || ((key >> hi) == prefix)) atomicAdd(&hist[(unsigned int)((key >> lo) & dmask)], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns bins 255-8l down to 248-8l (descending key order)
            unsigned int cnt[8], lsum = 0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                cnt[r] = hist[255 - 8 * lane - r];
                lsum += cnt[r];
            }
            unsigned int incl = lsum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned int y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const unsigned int excl = incl - lsum;
            const unsigned int krem = (unsigned int)sh_krem;
            if (excl < krem && krem <= incl) {  // exactly one lane
                unsigned int above = excl;
                int r = 0;
                while (above + cnt[r] < krem) {
                    above += cnt[r];
                    ++r;
                }
                const unsigned long long digit = 255u - 8u * lane - r;
                const unsigned int new_krem = krem - above;
                sh_prefix = (hi >= 64 ? 0ull : (prefix << (hi - lo))) | digit;
                sh_hi = lo;
                sh_krem = (int)new_krem;
                sh_done = (cnt[r] == new_krem) || lo == 0;
            }
        }
        __syncthreads();
    }
    const int fhi = sh_hi;
    const unsigned long long fprefix = sh_prefix;
    const bool keep_all = (m <= C);

    // ---- 2. kept flags: a key is kept iff its bits above fhi are at least
    // the threshold's (every key whose leading bits lie above the threshold's,
    // and the whole final bin)
    for (int c = threadIdx.x; c < m; c += blockDim.x) {
        const bool k = keep_all || fhi >= 64 || ((key_of(c) >> fhi) >= fprefix);
        skept[c] = (uint8_t)k;
        kept_g[c] = (uint8_t)k;
    }
    __syncthreads();

    // ---- 3. one scan for both: free slots (empty, or holding an evicted
    // entry) in ascending order, and kept chunk tokens in position order
    const int seg_c = (C + blockDim.x - 1) / blockDim.x;
    const int j0 = min(C, (int)threadIdx.x * seg_c), j1 = min(C, j0 + seg_c);
    const int seg_t = (T + blockDim.x - 1) / blockDim.x;
    const int t0 = min(T, (int)threadIdx.x * seg_t), t1 = min(T, t0 + seg_t);
    unsigned long long nfree_local = 0, nk_local = 0;
    for (int j = j0; j < j1; ++j) nfree_local += (j >= n || !skept[j]);
    for (int t = t0; t < t1; ++t) nk_local += skept[n + t];
    unsigned long long total;
    const unsigned long long ex =
        block_exclusive_scan<unsigned long long>((nfree_local << 32) | nk_local, scan_scratch, &total);
    const int n_free = (int)(total >> 32), n_tok = (int)(total & 0xffffffffull);
    int r = (int)(ex >> 32);
    for (int j = j0; j < j1; ++j)
        if (j >= n || !skept[j]) sfree[r++] = j;
    __syncthreads();

    // ---- 4. kept chunk tokens, in position order, take the free slots
    int rt = (int)(ex & 0xffffffffull);
    for (int t = t0; t < t1; ++t) {
        int slot = -1;
        if (skept[n + t] && rt < n_free) {
            slot = sfree[rt];
            sc[slot] = cs[n + t];
            ps[slot] = (int32_t)(P + t);
            stok[rt] = t;
        }
        rt += skept[n + t];
        ts[t] = slot;
    }
    // free slots nobody took stay (or become) empty
    for (int rr = n_tok + threadIdx.x; rr < n_free; rr += blockDim.x) {
        const int j = sfree[rr];
        sc[j] = 0.f;
        ps[j] = -1;
    }
    __syncthreads();  // the kept-token list is complete

    // ---- 5. copy the kept tokens' key and value rows into their slots (the
    // r-th kept token takes free slot r): a warp takes four list entries at a
    // time, 16 bytes per lane per access, every load of the four issued
    // before any store
    const int n_copy = min(n_tok, n_free);
    const int nwarps = (int)(blockDim.x >> 5);
    for (int r0 = 4 * warp; r0 < n_copy; r0 += 4 * nwarps) {
        int tk[4], sl[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool on = r0 + u < n_copy;
            tk[u] = on ? stok[r0 + u] : 0;
            sl[u] = on ? sfree[r0 + u] : -1;
        }
        for (int e0 = 0; e0 < row_vecs; e0 += 32) {
            const int e = e0 + lane;
            uint4 kx[4], vx[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (sl[u] >= 0 && e < row_vecs) {
                    const size_t src = (bg * T + tk[u]) * (size_t)row_vecs + e;
                    kx[u] = kin[src];
                    vx[u] = vin[src];
                }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (sl[u] >= 0 && e < row_vecs) {
                    const size_t dst = (bg * C + sl[u]) * (size_t)row_vecs + e;
                    Kc[dst] = kx[u];
                    Vc[dst] = vx[u];
                }
        }
    }
}

// One warp per chunk token row: copy its key and value rows into the slot
// chosen for it, 16 bytes per lane per access (insert-always; the other
// policies copy inside select_kernel).
__global__ void __launch_bounds__(256)
scatter_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ Kc,
               uint4* __restrict__ Vc, const int32_t* __restrict__ token_slot, int Hkv, int C, int T,
               int tmax, int row_vecs) {
    griddep_wait();  // the token -> slot map is written
    griddep_launch_dependents();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int t = blockIdx.x * 8 + warp;
    const size_t bg = (size_t)blockIdx.z * Hkv + blockIdx.y;
    if (t >= T) return;
    const int slot = token_slot[bg * tmax + t];
    if (slot < 0) return;
    const size_t src = (bg * T + t) * (size_t)row_vecs;
    const size_t dst = (bg * C + slot) * (size_t)row_vecs;
    for (int e = lane; e < row_vecs; e += 32) {
        Kc[dst + e] = k[src + e];
        Vc[dst + e] = v[src + e];
    }
}

__global__ void wait_selftest_kernel(WaitBound wb) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Nothing arrives on this barrier; the bounded wait must give up.
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, wb, kDevTimeoutSelftest);
    __syncthreads();
}

}  // namespace

// The selection and copy kernels are launched with programmatic dependent
// launch: their CTAs start (and fetch their code) while the previous kernel
// drains, then wait for it in griddep_wait().
constexpr bool kEarlyLaunch = true;

cudaError_t launch_select(const StepArgs& a) {
    const int m = a.n + a.T;
    // kept flags + free list + kept-token list
    const size_t tail = (((size_t)m + 15) & ~(size_t)15) + (size_t)a.C * 4 + (size_t)a.T * 4;
    const size_t with_keys = (size_t)m * 8 + tail;
    const int row_vecs = a.d * (a.dtype == 1 ? 4 : 2) / 16;
    if (cudaError_t e = ensure_smem_limit(select_kernel<true>, kSelectSmemLimit); e != cudaSuccess) return e;
    if (cudaError_t e = ensure_smem_limit(select_kernel<false>, kSelectSmemLimit); e != cudaSuccess) return e;
    const bool keys_fit = with_keys <= (size_t)kSelectSmemLimit;
    if (!keys_fit && tail > (size_t)kSelectSmemLimit) return cudaErrorInvalidConfiguration;
    cudaError_t e = launch_ex(kEarlyLaunch, keys_fit ? select_kernel<true> : select_kernel<false>, dim3(a.B * a.Hkv),
                              dim3(kSelThreads), keys_fit ? with_keys : tail, a.stream, a.cand_score, a.cand_pos,
                              a.cand_kept, a.token_slot, a.scores, a.pos, (const float*)a.partials, a.nparts, a.C,
                              a.T, a.n, a.tmax, (long long)a.P, a.policy, (const uint4*)a.k, (const uint4*)a.v,
                              (uint4*)a.Kc, (uint4*)a.Vc, row_vecs);
    if (e != cudaSuccess) return e;
    a.log->done("select_kernel", a.stream);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const StepArgs& a) {
    const int elem = a.dtype == 1 ? 4 : 2;
    const int row_vecs = a.d * elem / 16;
    dim3 grid((a.T + 7) / 8, a.Hkv, a.B);
    cudaError_t e = launch_ex(kEarlyLaunch, scatter_kernel, grid, dim3(256), 0, a.stream, (const uint4*)a.k, (const uint4*)a.v,
                               (uint4*)a.Kc, (uint4*)a.Vc, (const int32_t*)a.token_slot, a.Hkv, a.C, a.T, a.tmax,
                               row_vecs);
    if (e != cudaSuccess) return e;
    a.log->done("scatter_kernel", a.stream);
    return cudaGetLastError();
}

cudaError_t launch_wait_selftest(const WaitBound& wb, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(wb);
    return cudaGetLastError();
}

}  // namespace h2o
