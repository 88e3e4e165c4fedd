// insert.cu -- the insert-always variant of the step ("Learning how to
// Forget", paper page, section "Improvements to Heavy-Hitter Oracle (H2O)":
// new content overwrites the slots with the smallest scores; section
// "Kernel Support Needs": attention under the position mask).
//
// Reading: before the chunk attends, if the n valid entries and the T chunk
// tokens do not fit, the need = n + T - C valid slots with the lowest scores
// so far go (lowest first, the older position first among equal scores); the
// chunk tokens, in position order, take the empty and evicted slots in
// ascending slot order with score 0; every row then attends to the buffer
// (slot j visible to row i iff pos_j <= P + i) and every valid slot's score
// grows by the weights it receives. All T chunk tokens enter, so T <= C.
//
// On the device the attention over the buffer is the ordinary chunk step over
// a compact cache: the kept old entries (all positions < P, so visible to
// every row) as the cache part and the chunk as the causal part. The kernels
// here pick the kept set and the slots (insert_select_kernel), copy the kept
// rows to the compact buffers (gather_kernel), and after the SDPA and weight
// sums of the chunk path write the new scores and positions into the slot
// layout (insert_finish_kernel); the chunk path's copy kernel then writes the
// chunk's K and V into their slots.
#include "kernels.h"

namespace h2o {
namespace {

constexpr int kInsThreads = 1024;

__device__ __forceinline__ uint32_t ins_ordered_bits(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long ins_key(const float* sc, const int32_t* ps, int j) {
    return ((unsigned long long)ins_ordered_bits(sc[j]) << 32) | (uint32_t)ps[j];
}

// Exclusive prefix sum of one int per thread over the block (scratch >= 33).
__device__ int ins_block_scan(int v, int* scratch, int* total) {
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
        if (lane < nwarps) scratch[lane] = w;
        if (lane == 31) scratch[32] = w;
    }
    __syncthreads();
    const int base = warp > 0 ? scratch[warp - 1] : 0;
    *total = scratch[32];
    const int r = base + x - v;
    __syncthreads();
    return r;
}

// One CTA per (sequence, KV head). Keeps the n - need highest valid slots (by
// (score, position)), numbers the kept slots in ascending order (their index
// in the compact cache), and lists the free slots in ascending order; chunk
// token t goes to free slot t. Outputs: compact_slot [groups][C] (slot of
// compact entry r), compact_score / compact_pos [groups][C] (the kept entries'
// scores and positions, in compact order), token_slot [groups][tmax].
__global__ void __launch_bounds__(kInsThreads)
insert_select_kernel(const float* __restrict__ scores, const int32_t* __restrict__ pos,
                     int32_t* __restrict__ compact_slot, float* __restrict__ compact_score,
                     int32_t* __restrict__ compact_pos, int32_t* __restrict__ token_slot,
                     uint8_t* __restrict__ kept_out, int C, int T, int n, int tmax) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ unsigned int hist[256];
    __shared__ int scan_scratch[33];
    __shared__ unsigned long long sh_prefix;
    __shared__ int sh_shift, sh_krem, sh_done;
    extern __shared__ int32_t ins_free[];  // [C] free slots, ascending
    const size_t bg = blockIdx.x;
    const float* sc = scores + bg * (size_t)C;
    const int32_t* ps = pos + bg * (size_t)C;
    const int need = n + T - C;        // entries to evict (if positive)
    const int keep = need > 0 ? n - need : n;

    // threshold: the keep-th largest key among the n valid slots (MSB-first
    // radix select, 8 bits a pass, early exit when a bin holds exactly the rest)
    if (threadIdx.x == 0) {
        sh_prefix = 0ull;
        sh_shift = 64;
        sh_krem = keep;
        sh_done = need <= 0 || keep == 0;
    }
    __syncthreads();
    while (!sh_done) {
        const int shift = sh_shift - 8;
        const unsigned long long prefix = sh_prefix;
        for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0u;
        __syncthreads();
        for (int j = threadIdx.x; j < n; j += blockDim.x) {
            const unsigned long long key = ins_key(sc, ps, j);
            if (shift == 56 || (key >> (shift + 8)) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
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
            if (excl < krem && krem <= incl) {
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
    const bool all = need <= 0;

    // kept flags, compact numbering (ascending slots) and free slots (ascending)
    const int seg = (C + blockDim.x - 1) / blockDim.x;
    const int j0 = min(C, (int)threadIdx.x * seg), j1 = min(C, j0 + seg);
    auto kept = [&](int j) -> bool {
        if (j >= n) return false;
        if (all) return true;
        if (keep == 0) return false;
        return fshift >= 64 || (ins_key(sc, ps, j) >> fshift) >= fprefix;
    };
    int nk = 0, nf = 0;
    for (int j = j0; j < j1; ++j) {
        const bool k = kept(j);
        nk += k;
        nf += !k;
    }
    int tot_k, tot_f;
    int rk = ins_block_scan(nk, scan_scratch, &tot_k);
    int rf = ins_block_scan(nf, scan_scratch, &tot_f);
    for (int j = j0; j < j1; ++j) {
        if (kept(j)) {
            compact_slot[bg * (size_t)C + rk] = j;
            compact_score[bg * (size_t)C + rk] = sc[j];
            compact_pos[bg * (size_t)C + rk] = ps[j];
            ++rk;
        } else {
            ins_free[rf++] = j;
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) token_slot[bg * (size_t)tmax + t] = t < tot_f ? ins_free[t] : -1;
    // the step's candidates are the kept entries (compact order) and the chunk: all kept
    uint8_t* ko = kept_out + bg * (size_t)(C + tmax);
    for (int c = threadIdx.x; c < tot_k + T; c += blockDim.x) ko[c] = 1;
}

// One warp per compact entry r: copies the K and V rows of its slot.
__global__ void __launch_bounds__(256)
gather_kernel(const uint4* __restrict__ Kc, const uint4* __restrict__ Vc, uint4* __restrict__ Kq,
              uint4* __restrict__ Vq, const int32_t* __restrict__ compact_slot, int C, int n_kept,
              int row_vecs) {
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int r = blockIdx.x * 8 + warp;
    const size_t bg = blockIdx.y;
    if (r >= n_kept) return;
    const int j = compact_slot[bg * (size_t)C + r];
    const uint4* ks = Kc + (bg * C + j) * (size_t)row_vecs;
    const uint4* vs = Vc + (bg * C + j) * (size_t)row_vecs;
    uint4* kd = Kq + (bg * C + r) * (size_t)row_vecs;
    uint4* vd = Vq + (bg * C + r) * (size_t)row_vecs;
    for (int e = lane; e < row_vecs; e += 32) {
        kd[e] = ks[e];
        vd[e] = vs[e];
    }
}

// One CTA per group: the step's new scores into the slot layout. Compact entry
// r (slot compact_slot[r]) gets its old score plus the weight-sum partials of
// candidate r, in part order; chunk token t (candidate n_kept + t) goes to
// token_slot[t] with its weight sum and position P + t; slots left free (none
// when the chunk filled the cache) become empty.
__global__ void __launch_bounds__(256)
insert_finish_kernel(const int32_t* __restrict__ compact_slot, const float* __restrict__ compact_score,
                     const int32_t* __restrict__ token_slot, const float* __restrict__ partials, int nparts,
                     const float* __restrict__ cand_direct, float* __restrict__ scores, int32_t* __restrict__ pos,
                     float* __restrict__ cand_score, int32_t* __restrict__ cand_pos,
                     const int32_t* __restrict__ compact_pos, int C, int T, int n_kept, int tmax,
                     long long P) {
    griddep_wait();
    griddep_launch_dependents();
    const size_t bg = blockIdx.x;
    const size_t cstride = (size_t)C + tmax;
    const size_t pstride = (size_t)gridDim.x * cstride;
    for (int c = threadIdx.x; c < n_kept + T; c += blockDim.x) {
        float s;
        if (nparts > 0) {
            s = c < n_kept ? compact_score[bg * (size_t)C + c] : 0.f;
            for (int q = 0; q < nparts; ++q) s += partials[q * pstride + bg * cstride + c];
        } else {
            s = cand_direct[bg * cstride + c];  // the CUDA-core weight sums wrote old + delta
        }
        const int32_t p = c < n_kept ? compact_pos[bg * (size_t)C + c] : (int32_t)(P + (c - n_kept));
        cand_score[bg * cstride + c] = s;
        cand_pos[bg * cstride + c] = p;
        const int slot = c < n_kept ? compact_slot[bg * (size_t)C + c] : token_slot[bg * (size_t)tmax + (c - n_kept)];
        if (slot >= 0) {
            scores[bg * (size_t)C + slot] = s;
            pos[bg * (size_t)C + slot] = p;
        }
    }
}

}  // namespace

cudaError_t launch_insert_select(const StepArgs& a, int n_kept) {
    const size_t smem = sizeof(int32_t) * (size_t)a.C;
    if (smem > 48 * 1024) {
        if (cudaError_t e = ensure_smem_limit(insert_select_kernel, 227 * 1024); e != cudaSuccess) return e;
    }
    (void)n_kept;
    cudaError_t e = launch_ex(true, insert_select_kernel, dim3(a.B * a.Hkv), dim3(kInsThreads), smem, a.stream,
                              (const float*)a.scores, (const int32_t*)a.pos, a.ins_slot, a.ins_score, a.ins_pos,
                              a.token_slot, a.cand_kept, a.C, a.T, a.n, a.tmax);
    if (e != cudaSuccess) return e;
    a.log->done("insert_select_kernel", a.stream);
    return cudaGetLastError();
}

cudaError_t launch_gather(const StepArgs& a, int n_kept) {
    if (n_kept == 0) return cudaSuccess;
    const int elem = a.dtype == 1 ? 4 : 2;
    const int row_vecs = a.d * elem / 16;
    cudaError_t e = launch_ex(true, gather_kernel, dim3((n_kept + 7) / 8, a.B * a.Hkv), dim3(256), 0, a.stream,
                              (const uint4*)a.Kc, (const uint4*)a.Vc, (uint4*)a.ins_K, (uint4*)a.ins_V,
                              (const int32_t*)a.ins_slot, a.C, n_kept, row_vecs);
    if (e != cudaSuccess) return e;
    a.log->done("gather_kernel", a.stream);
    return cudaGetLastError();
}

cudaError_t launch_insert_finish(const StepArgs& a, int n_kept) {
    cudaError_t e = launch_ex(true, insert_finish_kernel, dim3(a.B * a.Hkv), dim3(256), 0, a.stream,
                              (const int32_t*)a.ins_slot, (const float*)a.ins_score, (const int32_t*)a.token_slot,
                              (const float*)a.partials, a.nparts, (const float*)a.cand_score, a.scores, a.pos,
                              a.cand_score, a.cand_pos, (const int32_t*)a.ins_pos, a.C, a.T, n_kept, a.tmax,
                              (long long)a.P);
    if (e != cudaSuccess) return e;
    a.log->done("insert_finish_kernel", a.stream);
    return cudaGetLastError();
}

}  // namespace h2o
