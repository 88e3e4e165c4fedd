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
// to slot map. The key/value copy is a separate wide grid of 16-byte vector
// copies so that HBM bandwidth, not the handful of selection CTAs, bounds it.
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

__device__ __forceinline__ uint64_t cand_key(const float* cs, const int32_t* cp, int c) {
    return ((uint64_t)ordered_bits(cs[c]) << 32) | (uint32_t)cp[c];
}

// Candidate keys are staged in shared memory when they fit (the radix passes
// then read them from there), otherwise rebuilt from global memory per pass.
constexpr int kSmemKeyLimit = 24576;  // 192 KB of 64-bit keys

// Exclusive prefix sum of one int per thread over the block; *total gets the
// sum. Uses `scratch` (>= 33 ints of shared memory).
__device__ int block_exclusive_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? scratch[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < nwarps) scratch[lane] = w;  // inclusive warp totals
        if (lane == 31) scratch[32] = w;
    }
    __syncthreads();
    const int base = warp > 0 ? scratch[warp - 1] : 0;
    *total = scratch[32];
    const int r = base + x - v;
    __syncthreads();
    return r;
}

template <bool SMEM_KEYS>
__global__ void __launch_bounds__(kSelThreads)
select_kernel(float* __restrict__ cand_score, int32_t* __restrict__ cand_pos,
              uint8_t* __restrict__ cand_kept, int32_t* __restrict__ token_slot,
              int32_t* __restrict__ free_list, float* __restrict__ scores, int32_t* __restrict__ pos,
              const float* __restrict__ partials, int nparts, int C, int T, int n, int tmax, long long P) {
    __shared__ unsigned int hist[256];
    __shared__ int scan_scratch[33];
    __shared__ unsigned long long sh_prefix;
    __shared__ int sh_shift, sh_krem, sh_done;
    extern __shared__ unsigned long long skeys[];  // [m] when SMEM_KEYS

    const size_t bg = blockIdx.x;
    const int m = n + T;
    float* cs = cand_score + bg * (size_t)(C + tmax);
    int32_t* cp = cand_pos + bg * (size_t)(C + tmax);
    uint8_t* kept = cand_kept + bg * (size_t)(C + tmax);
    int32_t* fl = free_list + bg * (size_t)C;
    int32_t* ts = token_slot + bg * (size_t)tmax;
    float* sc = scores + bg * (size_t)C;
    int32_t* ps = pos + bg * (size_t)C;

    // ---- 0. candidate scores from the weight-sum partials (fixed part order)
    if (nparts > 0) {
        const size_t pstride = (size_t)gridDim.x * (C + tmax);
        for (int c = threadIdx.x; c < m; c += blockDim.x) {
            float s = c < n ? sc[c] : 0.f;
            for (int q = 0; q < nparts; ++q) s += partials[q * pstride + bg * (size_t)(C + tmax) + c];
            cs[c] = s;
            cp[c] = c < n ? ps[c] : (int32_t)(P + (c - n));
        }
        __syncthreads();
    }
    if (SMEM_KEYS) {
        for (int c = threadIdx.x; c < m; c += blockDim.x) skeys[c] = cand_key(cs, cp, c);
        __syncthreads();
    }
    auto key_of = [&](int c) -> uint64_t { return SMEM_KEYS ? (uint64_t)skeys[c] : cand_key(cs, cp, c); };

    // ---- 1. threshold: the C-th largest key (radix select, 8 bits a pass)
    if (threadIdx.x == 0) {
        sh_prefix = 0ull;
        sh_shift = 64;
        sh_krem = C;
        sh_done = (m <= C);
    }
    __syncthreads();
    while (!sh_done) {
        const int shift = sh_shift - 8;
        const unsigned long long prefix = sh_prefix;
        for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0u;
        __syncthreads();
        for (int c = threadIdx.x; c < m; c += blockDim.x) {
            const uint64_t key = key_of(c);
            const bool match = (shift == 56) || ((key >> (shift + 8)) == prefix);
            if (match) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns bins 255-8l down to 248-8l (descending key order)
            const int lane = threadIdx.x;
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
                const unsigned int digit = 255u - 8u * lane - r;
                const unsigned int new_krem = krem - above;
                sh_prefix = (prefix << 8) | digit;
                sh_shift = shift;
                sh_krem = (int)new_krem;
                sh_done = (cnt[r] == new_krem) || shift == 0;
            }
        }
        __syncthreads();
    }
    const int fshift = sh_shift;
    const unsigned long long fprefix = sh_prefix;
    const bool keep_all = (m <= C);

    // ---- 2. kept flags
    for (int c = threadIdx.x; c < m; c += blockDim.x) {
        bool k = keep_all;
        if (!keep_all) {
            const uint64_t key = key_of(c);
            k = fshift >= 64 ? true : ((key >> fshift) >= fprefix);
        }
        kept[c] = (uint8_t)k;
    }
    __syncthreads();

    // ---- 3. free slots (empty, or holding an evicted entry), ascending
    const int seg_c = (C + blockDim.x - 1) / blockDim.x;
    const int j0 = min(C, (int)threadIdx.x * seg_c), j1 = min(C, j0 + seg_c);
    int nfree_local = 0;
    for (int j = j0; j < j1; ++j) nfree_local += (j >= n || !kept[j]);
    int n_free;
    int r = block_exclusive_scan(nfree_local, scan_scratch, &n_free);
    for (int j = j0; j < j1; ++j) {
        if (j >= n || !kept[j]) fl[r++] = j;
        else sc[j] = cs[j];  // kept cache slot: its updated score
    }
    __syncthreads();

    // ---- 4. kept chunk tokens, in position order, take the free slots
    const int seg_t = (T + blockDim.x - 1) / blockDim.x;
    const int t0 = min(T, (int)threadIdx.x * seg_t), t1 = min(T, t0 + seg_t);
    int nk_local = 0;
    for (int t = t0; t < t1; ++t) nk_local += kept[n + t];
    int n_tok;
    int rt = block_exclusive_scan(nk_local, scan_scratch, &n_tok);
    for (int t = t0; t < t1; ++t) {
        int slot = -1;
        if (kept[n + t] && rt < n_free) {
            slot = fl[rt];
            sc[slot] = cs[n + t];
            ps[slot] = (int32_t)(P + t);
        }
        rt += kept[n + t];
        ts[t] = slot;
    }
    // free slots nobody took stay (or become) empty
    for (int rr = n_tok + threadIdx.x; rr < n_free; rr += blockDim.x) {
        const int j = fl[rr];
        sc[j] = 0.f;
        ps[j] = -1;
    }
}

// One warp per chunk token row: copy its key and value rows into the slot
// chosen for it, 16 bytes per lane per access.
__global__ void __launch_bounds__(256)
scatter_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ Kc,
               uint4* __restrict__ Vc, const int32_t* __restrict__ token_slot, int Hkv, int C, int T,
               int tmax, int row_vecs) {
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

cudaError_t launch_select(const StepArgs& a) {
    const int m = a.n + a.T;
    if (m <= kSmemKeyLimit) {
        static int configured = 0;
        if (!configured) {
            cudaError_t e = cudaFuncSetAttribute(select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemKeyLimit * 8);
            if (e != cudaSuccess) return e;
            configured = 1;
        }
        select_kernel<true><<<a.B * a.Hkv, kSelThreads, (size_t)m * 8, a.stream>>>(
            a.cand_score, a.cand_pos, a.cand_kept, a.token_slot, a.free_list, a.scores, a.pos, a.partials,
            a.nparts, a.C, a.T, a.n, a.tmax, (long long)a.P);
    } else {
        select_kernel<false><<<a.B * a.Hkv, kSelThreads, 0, a.stream>>>(
            a.cand_score, a.cand_pos, a.cand_kept, a.token_slot, a.free_list, a.scores, a.pos, a.partials,
            a.nparts, a.C, a.T, a.n, a.tmax, (long long)a.P);
    }
    a.log->done("select_kernel", a.stream);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const StepArgs& a) {
    const int elem = a.dtype == 1 ? 4 : 2;
    const int row_vecs = a.d * elem / 16;
    dim3 grid((a.T + 7) / 8, a.Hkv, a.B);
    scatter_kernel<<<grid, 256, 0, a.stream>>>((const uint4*)a.k, (const uint4*)a.v, (uint4*)a.Kc,
                                               (uint4*)a.Vc, a.token_slot, a.Hkv, a.C, a.T, a.tmax,
                                               row_vecs);
    a.log->done("scatter_kernel", a.stream);
    return cudaGetLastError();
}

cudaError_t launch_wait_selftest(const WaitBound& wb, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(wb);
    return cudaGetLastError();
}

}  // namespace h2o
