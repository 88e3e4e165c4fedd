// simt.cu -- SIMT (CUDA-core) kernels of the H2O step: chunk SDPA with the
// per-row log-sum-exp, and the per-key attention-weight sums.
//
// These carry the fp32 path, where tensor-core tf32 rounding would exceed the
// fp32 tolerance, and any shape the tensor-core kernels do not take. The
// arithmetic is fp32 throughout.
//
// What they compute ("Learning how to Forget", paper page, sections "Kernel
// Support Needs" and "Improvements to Heavy-Hitter Oracle (H2O)"): for every
// query row i of head h (position P+i) the softmax over the keys whose
// position is <= P+i -- all n valid cache slots and the chunk tokens t <= i --
// of scale * q.k, the output sum_j w_j v_j and LSE = log sum_j exp(logit_j);
// then for every key c of KV head g the sum over the group's heads and rows
// of exp(scale * q.k_c - LSE) over the rows that see c.
#include "kernels.h"

namespace h2o {
namespace {

constexpr int kRowsPerBlock = 4;   // one warp per query row
constexpr int kKeyTile = 32;       // one lane per key in a tile

template <typename E, int D>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
sdpa_simt_kernel(const E* __restrict__ q, const E* __restrict__ Kc, const E* __restrict__ Vc,
                 const E* __restrict__ k, const E* __restrict__ v, E* __restrict__ out,
                 float* __restrict__ lse, int Hq, int Hkv, int C, int T, int n, int tmax,
                 float scale_log2) {
    __shared__ float Ks[kKeyTile][D + 1];
    __shared__ float Vs[kKeyTile][D];
    __shared__ float Qs[kRowsPerBlock][D];
    constexpr int PER_LANE = D / 32;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int h = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    const size_t bg = (size_t)b * Hkv + h / G;
    const int i0 = blockIdx.x * kRowsPerBlock;
    const int i = i0 + warp;
    const bool row_ok = i < T;
    const size_t qrow = ((size_t)b * Hq + h) * T + (row_ok ? i : 0);

    for (int x = lane; x < D; x += 32) Qs[warp][x] = row_ok ? to_f32(q[qrow * D + x]) : 0.f;

    // keys u in [0, n + T): u < n is cache slot u, otherwise chunk token u - n
    const int i_last = min(i0 + kRowsPerBlock, T) - 1;
    const int n_keys = n + i_last + 1;
    float m = -INFINITY, l = 0.f;
    float o[PER_LANE];
#pragma unroll
    for (int r = 0; r < PER_LANE; ++r) o[r] = 0.f;

    for (int u0 = 0; u0 < n_keys; u0 += kKeyTile) {
        __syncthreads();
        for (int e = threadIdx.x; e < kKeyTile * D; e += blockDim.x) {
            const int j = e / D, x = e % D, u = u0 + j;
            float kv = 0.f, vv = 0.f;
            if (u < n) {
                kv = to_f32(Kc[(bg * C + u) * D + x]);
                vv = to_f32(Vc[(bg * C + u) * D + x]);
            } else if (u < n_keys) {
                kv = to_f32(k[(bg * T + (u - n)) * D + x]);
                vv = to_f32(v[(bg * T + (u - n)) * D + x]);
            }
            Ks[j][x] = kv;
            Vs[j][x] = vv;
        }
        __syncthreads();
        const int u = u0 + lane;
        const bool vis = row_ok && (u < n || (u < n_keys && u - n <= i));
        float s = -INFINITY;
        if (vis) {
            float acc = 0.f;
#pragma unroll 8
            for (int x = 0; x < D; ++x) acc = fmaf(Qs[warp][x], Ks[lane][x], acc);
            s = acc * scale_log2;
        }
        float tmax_s = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) tmax_s = fmaxf(tmax_s, __shfl_xor_sync(0xffffffffu, tmax_s, off));
        const float m_new = fmaxf(m, tmax_s);
        if (m_new == -INFINITY) continue;  // nothing visible yet in this row (uniform per warp)
        const float corr = exp2f(m - m_new);
        const float p = vis ? exp2f(s - m_new) : 0.f;
        float psum = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l = l * corr + psum;
#pragma unroll
        for (int r = 0; r < PER_LANE; ++r) o[r] *= corr;
        for (int j = 0; j < kKeyTile; ++j) {
            const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
            for (int r = 0; r < PER_LANE; ++r) o[r] = fmaf(pj, Vs[j][lane + 32 * r], o[r]);
        }
        m = m_new;
    }
    if (row_ok) {
        const float inv = 1.f / l;
#pragma unroll
        for (int r = 0; r < PER_LANE; ++r) out[qrow * D + lane + 32 * r] = from_f32<E>(o[r] * inv);
        if (lane == 0) lse[((size_t)b * Hq + h) * tmax + i] = (m + log2f(l)) * kLn2;
    }
}

constexpr int kKeysPerBlock = 128;  // one thread per candidate key
constexpr int kRowTile = 32;

template <typename E, int D>
__global__ void __launch_bounds__(kKeysPerBlock)
wsum_simt_kernel(const E* __restrict__ q, const E* __restrict__ Kc, const E* __restrict__ k,
                 const float* __restrict__ lse, const float* __restrict__ scores,
                 const int32_t* __restrict__ pos, float* __restrict__ cand_score,
                 int32_t* __restrict__ cand_pos, int Hq, int Hkv, int C, int T, int n, int tmax,
                 long long P, float scale_log2) {
    extern __shared__ float smem[];
    float* Ks = smem;                                  // [kKeysPerBlock][D+1]
    float* Qs = Ks + kKeysPerBlock * (D + 1);          // [kRowTile][D]
    float* L2s = Qs + kRowTile * D;                    // [kRowTile]

    const int g = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    const size_t bg = (size_t)b * Hkv + g;
    const int c0 = blockIdx.x * kKeysPerBlock;
    const int c = c0 + threadIdx.x;
    const int n_cand = n + T;
    const bool ok = c < n_cand;

    for (int e = threadIdx.x; e < kKeysPerBlock * D; e += blockDim.x) {
        const int j = e / D, x = e % D, cc = c0 + j;
        float kv = 0.f;
        if (cc < n) kv = to_f32(Kc[(bg * C + cc) * D + x]);
        else if (cc < n_cand) kv = to_f32(k[(bg * T + (cc - n)) * D + x]);
        Ks[j * (D + 1) + x] = kv;
    }
    // the first row that sees any key of this block: 0 if it holds a cache
    // slot, otherwise the first chunk token's own row
    const int first_row = (c0 < n) ? 0 : (c0 - n);
    const int t_self = c - n;  // chunk token index (negative for cache slots)
    float acc = 0.f;
    for (int hh = 0; hh < G; ++hh) {
        const size_t qh = (size_t)b * Hq + (size_t)g * G + hh;
        for (int i0 = (first_row / kRowTile) * kRowTile; i0 < T; i0 += kRowTile) {
            __syncthreads();
            for (int e = threadIdx.x; e < kRowTile * D; e += blockDim.x) {
                const int r = e / D, x = e % D, i = i0 + r;
                Qs[e] = (i < T) ? to_f32(q[(qh * T + i) * D + x]) : 0.f;
            }
            if (threadIdx.x < kRowTile) {
                const int i = i0 + threadIdx.x;
                L2s[threadIdx.x] = (i < T) ? lse[qh * tmax + i] * kLog2e : 0.f;
            }
            __syncthreads();
            if (!ok) continue;
            for (int r = 0; r < kRowTile; ++r) {
                const int i = i0 + r;
                if (i >= T || i < t_self) continue;  // row does not see this key
                float dot = 0.f;
#pragma unroll 8
                for (int x = 0; x < D; ++x) dot = fmaf(Qs[r * D + x], Ks[threadIdx.x * (D + 1) + x], dot);
                acc += exp2f(fmaf(dot, scale_log2, -L2s[r]));
            }
        }
    }
    if (ok) {
        const size_t o = bg * (size_t)(C + tmax) + c;
        if (c < n) {
            cand_score[o] = scores[bg * C + c] + acc;
            cand_pos[o] = pos[bg * C + c];
        } else {
            cand_score[o] = acc;
            cand_pos[o] = (int32_t)(P + (c - n));
        }
    }
}

template <typename E, int D>
cudaError_t sdpa_simt_typed(const StepArgs& a) {
    dim3 grid((a.T + kRowsPerBlock - 1) / kRowsPerBlock, a.Hq, a.B);
    const float scale_log2 = kLog2e / sqrtf((float)D);
    sdpa_simt_kernel<E, D><<<grid, kRowsPerBlock * 32, 0, a.stream>>>(
        (const E*)a.q, (const E*)a.Kc, (const E*)a.Vc, (const E*)a.k, (const E*)a.v, (E*)a.out, a.lse,
        a.Hq, a.Hkv, a.C, a.T, a.n, a.tmax, scale_log2);
    a.log->done("sdpa_simt_kernel", a.stream);
    return cudaGetLastError();
}

template <typename E, int D>
cudaError_t wsum_simt_typed(const StepArgs& a) {
    const int n_cand = a.n + a.T;
    dim3 grid((n_cand + kKeysPerBlock - 1) / kKeysPerBlock, a.Hkv, a.B);
    const size_t smem = sizeof(float) * (kKeysPerBlock * (D + 1) + kRowTile * D + kRowTile);
    auto kern = wsum_simt_kernel<E, D>;
    cudaError_t e = ensure_smem_limit(kern, (int)smem);
    if (e != cudaSuccess) return e;
    const float scale_log2 = kLog2e / sqrtf((float)D);
    kern<<<grid, kKeysPerBlock, smem, a.stream>>>(
        (const E*)a.q, (const E*)a.Kc, (const E*)a.k, a.lse, a.scores, a.pos, a.cand_score, a.cand_pos,
        a.Hq, a.Hkv, a.C, a.T, a.n, a.tmax, (long long)a.P, scale_log2);
    a.log->done("wsum_simt_kernel", a.stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sdpa_simt(const StepArgs& a) {
    if (a.dtype == 1) return a.d == 64 ? sdpa_simt_typed<float, 64>(a) : sdpa_simt_typed<float, 128>(a);
    return a.d == 64 ? sdpa_simt_typed<__nv_bfloat16, 64>(a) : sdpa_simt_typed<__nv_bfloat16, 128>(a);
}

cudaError_t launch_wsum_simt(const StepArgs& a) {
    if (a.dtype == 1) return a.d == 64 ? wsum_simt_typed<float, 64>(a) : wsum_simt_typed<float, 128>(a);
    return a.d == 64 ? wsum_simt_typed<__nv_bfloat16, 64>(a) : wsum_simt_typed<__nv_bfloat16, 128>(a);
}

}  // namespace h2o
