// noalloc.cu -- eviction (selection + slot placement) without any device
// allocation, for callers that cannot call cudaMalloc.
//
// Some callers of this library cannot allocate device memory themselves:
// plugin hosts and serving runtimes that hand a plugin only the buffers they
// pre-allocated under a fixed memory budget, or latency-critical paths where a
// cudaMalloc would synchronise the device and stall unrelated streams. The
// regular path keeps its scratch (the free-slot list) in a buffer that
// h2o_create allocates; this entry point instead keeps it in a fixed-size
// array in the library's own device image, so a call needs nothing beyond the
// caller's inputs and outputs.
//
// The scratch array is a file-scope __device__ object: every GPU that loads
// the library holds it (kNoAllocScratchInts int32, 1 MiB) until the process
// exits, whether or not the entry point is ever called.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/h2o.h"
#include "kernels.h"

namespace {

constexpr int kNoAllocScratchInts = 1 << 18;  // free-slot list capacity: groups * C <= 262144
constexpr int kMaxDevices = 64;
constexpr int kThreads = 1024;

// Free-slot lists of all groups of one call. Shared by every call on a device;
// it keeps whatever the last call left in it. Nothing in it needs clearing:
// a call writes every entry it reads before reading it.
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchInts];

// Device address of g_noalloc_scratch per device (host code cannot use the
// symbol itself as a device pointer), with the CUDA context it was looked up
// in: after a device reset the library's module is loaded again in a new
// context, possibly at another address, so a changed context means a new
// lookup.
int32_t* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The driver's cuCtxGetCurrent, fetched through the runtime (the library
// does not link the driver API); nullptr if unavailable.
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}


__device__ __forceinline__ uint32_t na_ordered_bits(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t na_key(const float* cs, const int32_t* cp, int c) {
    return ((uint64_t)na_ordered_bits(cs[c]) << 32) | (uint32_t)cp[c];
}

// Block-wide exclusive prefix sum (one value per thread), total in *total.
__device__ int na_block_scan(int v, int* sm, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? sm[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nw) sm[lane] = w;
        if (lane == 31) sm[32] = w;
    }
    __syncthreads();
    const int r = (warp ? sm[warp - 1] : 0) + x - v;
    *total = sm[32];
    __syncthreads();
    return r;
}

// One block per group. Candidates are dense: [groups, n+T], cache slots
// 0..n-1 first, then the chunk tokens. The free-slot list of the group lives
// in the scratch array at free_list + group * C.
__global__ void __launch_bounds__(kThreads)
select_noalloc_kernel(const float* __restrict__ cand_score, const int32_t* __restrict__ cand_pos,
                      uint8_t* __restrict__ kept_out, int32_t* __restrict__ token_slot,
                      float* __restrict__ scores, int32_t* __restrict__ positions,
                      int32_t* __restrict__ free_list, int C, int n, int T, long long P) {
    __shared__ unsigned int hist[256];
    __shared__ int scan_sm[33];
    __shared__ unsigned long long s_prefix;
    __shared__ int s_shift, s_krem, s_done;

    const size_t g = blockIdx.x;
    const int m = n + T;
    const float* cs = cand_score + g * (size_t)m;
    const int32_t* cp = cand_pos + g * (size_t)m;
    uint8_t* kept = kept_out + g * (size_t)m;
    int32_t* fl = free_list + g * (size_t)C;
    int32_t* ts = token_slot + g * (size_t)T;
    float* sc = scores + g * (size_t)C;
    int32_t* ps = positions + g * (size_t)C;

    if (threadIdx.x == 0) {
        s_prefix = 0ull;
        s_shift = 64;
        s_krem = C;
        s_done = (m <= C);
    }
    __syncthreads();
    // MSB-first radix select of the C-th largest (score, position) key
    while (!s_done) {
        const int shift = s_shift - 8;
        const unsigned long long prefix = s_prefix;
        for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0u;
        __syncthreads();
        for (int c = threadIdx.x; c < m; c += blockDim.x) {
            const uint64_t key = na_key(cs, cp, c);
            if (shift == 56 || (key >> (shift + 8)) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            unsigned int cnt[8], sum = 0;
            for (int r = 0; r < 8; ++r) {
                cnt[r] = hist[255 - 8 * lane - r];
                sum += cnt[r];
            }
            unsigned int incl = sum;
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned int excl = incl - sum, krem = (unsigned int)s_krem;
            if (excl < krem && krem <= incl) {
                unsigned int above = excl;
                int r = 0;
                while (above + cnt[r] < krem) above += cnt[r++];
                const unsigned int left = krem - above;
                s_prefix = (prefix << 8) | (255u - 8u * lane - r);
                s_shift = shift;
                s_krem = (int)left;
                s_done = (cnt[r] == left) || shift == 0;
            }
        }
        __syncthreads();
    }
    const bool all = (m <= C);
    const int fshift = s_shift;
    const unsigned long long fprefix = s_prefix;
    for (int c = threadIdx.x; c < m; c += blockDim.x)
        kept[c] = (uint8_t)(all || fshift >= 64 || (na_key(cs, cp, c) >> fshift) >= fprefix);
    __syncthreads();

    // free slots ascending -> scratch list; kept cache slots take their new score
    const int seg = (C + blockDim.x - 1) / blockDim.x;
    const int j0 = min(C, (int)threadIdx.x * seg), j1 = min(C, j0 + seg);
    int local = 0;
    for (int j = j0; j < j1; ++j) local += (j >= n || !kept[j]);
    int n_free;
    int r = na_block_scan(local, scan_sm, &n_free);
    for (int j = j0; j < j1; ++j) {
        if (j >= n || !kept[j]) fl[r++] = j;
        else sc[j] = cs[j];
    }
    __syncthreads();

    // kept chunk tokens in position order take the free slots in order
    const int segt = (T + blockDim.x - 1) / blockDim.x;
    const int t0 = min(T, (int)threadIdx.x * segt), t1 = min(T, t0 + segt);
    int kl = 0;
    for (int t = t0; t < t1; ++t) kl += kept[n + t];
    int n_tok;
    int rt = na_block_scan(kl, scan_sm, &n_tok);
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
    for (int rr = n_tok + threadIdx.x; rr < n_free; rr += blockDim.x) {
        const int j = fl[rr];
        sc[j] = 0.f;
        ps[j] = -1;
    }
}

int na_fail(int code, const char* msg) {
    h2o::set_thread_error_message(msg);  // what h2o_last_error(NULL) reports
    return code;
}

// Device address of the scratch array on the current device; looked up once
// per device and context (the first call on a device does it, and the first
// call after the device's context changed, e.g. after cudaDeviceReset).
int scratch_address(int32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return na_fail(H2O_ERR_CUDA, "h2o_select_noalloc: cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices) return na_fail(H2O_ERR_UNSUPPORTED, "h2o_select_noalloc: device index too large");
    CtxGetCurrentFn get = ctx_get_current_fn();
    CUcontext ctx = nullptr;
    if (get && get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr || ctx == nullptr || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the context current
        if (e != cudaSuccess || p == nullptr)
            return na_fail(H2O_ERR_CUDA, "h2o_select_noalloc: cudaGetSymbolAddress of the scratch array failed");
        if (get && get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
        g_scratch_addr[dev] = static_cast<int32_t*>(p);
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_addr[dev];
    return H2O_OK;
}

}  // namespace

extern "C" {

int h2o_select_noalloc(int groups, int C, int n, int T, int64_t P, const float* cand_score,
                       const int32_t* cand_pos, float* scores, int32_t* positions, uint8_t* kept,
                       int32_t* token_slot, void* stream) {
    if (groups < 1 || C < 1 || T < 1 || n < 0 || n > C || P < 0 || P + T > (int64_t)INT32_MAX)
        return na_fail(H2O_ERR_ARG, "h2o_select_noalloc: need groups, C, T >= 1, 0 <= n <= C, P >= 0, P+T < 2^31");
    if (!cand_score || !cand_pos || !scores || !positions || !kept || !token_slot)
        return na_fail(H2O_ERR_ARG, "h2o_select_noalloc: a pointer argument is NULL");
    if ((long long)groups * C > kNoAllocScratchInts)
        return na_fail(H2O_ERR_UNSUPPORTED,
                       "h2o_select_noalloc: groups * C exceeds the built-in scratch of 262144 slots");
    int32_t* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != H2O_OK) return rc;
    select_noalloc_kernel<<<groups, kThreads, 0, (cudaStream_t)stream>>>(
        cand_score, cand_pos, kept, token_slot, scores, positions, scratch, C, n, T, (long long)P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return na_fail(H2O_ERR_CUDA, "h2o_select_noalloc: kernel launch failed");
    return H2O_OK;
}

}  // extern "C"
