// backward.cu -- CUDA-core kernels of the backward of one step's chunk SDPA
// with the step's key set held fixed (the replay of a logged step).
//
// "Learning how to Forget", paper page, section "Gradient Computation
// Strategy for Sparse Attention": the model is fine-tuned through the sparse
// cache, with every eviction decision of the forward pass logged and replayed
// in the backward pass, so the attention of a step is differentiated for the
// key set the step actually used. Per query row i of head h (positions of
// the keys as in the forward: every valid cache slot, and the chunk tokens
// t <= i):
//   p_j = exp(scale * q_i . k_j - LSE_i),   dp_j = dO_i . v_j,
//   D_i = sum_j p_j dp_j,                   ds_j = p_j (dp_j - D_i),
//   dq_i = scale * sum_j ds_j k_j,  dk_j += scale * ds_j q_i,  dv_j += p_j dO_i,
// a KV head's key and value gradients summing over the query heads of its
// group. The eviction is a discrete choice and carries no gradient.
// D_i (which equals dO_i . O_i) is accumulated from the recomputed p and dp
// rather than from the forward's output, which the bf16 path holds only
// rounded to bf16, and it is taken as sum_j p_j dp_j / sum_j p_j: with the
// forward's LSE off by a rounding-level e, every p_j is off by the factor e^-e,
// and dividing by sum_j p_j keeps sum_j ds_j = 0 exactly, so the error stays a
// factor near 1 instead of a term e * D_i * sum_j p_j k_j. dq_i then comes out
// of one pass over the keys as scale * (sum_j p_j dp_j k_j - D_i sum_j p_j k_j).
//
// These kernels carry the fp32 path (and any context without the tensor-core
// path) and compute in fp32; backward_tc.cu holds the tcgen05 kernels of the
// bf16 path.
#include "kernels.h"

namespace h2o {
namespace {

constexpr int kRowsPerBlock = 4;   // dq: one warp per query row
constexpr int kKeyTile = 32;       // one lane per key in a tile

// dq of kRowsPerBlock rows of one head, and the rows' D_i and log2-domain
// LSE for the key-gradient kernel: keys in tiles of 32 staged in shared
// memory, one lane per key for the dot products, then every lane adds its
// d / 32 columns of sum_j p_j dp_j k_j and sum_j p_j k_j.
template <typename E, int D>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
bwd_dq_simt_kernel(const E* __restrict__ q, const E* __restrict__ Kc, const E* __restrict__ Vc,
                   const E* __restrict__ k, const E* __restrict__ v, const E* __restrict__ dout,
                   const float* __restrict__ lse, float* __restrict__ Drow, float* __restrict__ L2row,
                   float* __restrict__ dq, int Hq, int Hkv, int C, int T, int n, int rows_pad, float scale_log2,
                   float scale) {
    __shared__ float Ks[kKeyTile][D + 1];
    __shared__ float Vs[kKeyTile][D + 1];
    __shared__ float Qs[kRowsPerBlock][D];
    __shared__ float Os[kRowsPerBlock][D];
    constexpr int PER_LANE = D / 32;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int h = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    const size_t bg = (size_t)b * Hkv + h / G;
    const int i0 = blockIdx.x * kRowsPerBlock;
    const int i = i0 + warp;
    const bool row_ok = i < T;
    const size_t qrow = ((size_t)b * Hq + h) * T + (row_ok ? i : 0);
    for (int x = lane; x < D; x += 32) {
        Qs[warp][x] = row_ok ? to_f32(q[qrow * D + x]) : 0.f;
        Os[warp][x] = row_ok ? to_f32(dout[qrow * D + x]) : 0.f;
    }
    const float L2 = row_ok ? lse[qrow] * kLog2e : 0.f;
    const int i_last = min(i0 + kRowsPerBlock, T) - 1;
    const int n_keys = n + i_last + 1;  // key u < n: cache slot u, else chunk token u - n
    float ga[PER_LANE], gb[PER_LANE];   // sum p dp k, sum p k (this lane's columns)
    float Dacc = 0.f, Pacc = 0.f;       // sum p dp, sum p over this lane's keys
#pragma unroll
    for (int r = 0; r < PER_LANE; ++r) ga[r] = gb[r] = 0.f;
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
        float p = 0.f, pdp = 0.f;
        if (vis) {
            float s = 0.f, dp = 0.f;
#pragma unroll 8
            for (int x = 0; x < D; ++x) {
                s = fmaf(Qs[warp][x], Ks[lane][x], s);
                dp = fmaf(Os[warp][x], Vs[lane][x], dp);
            }
            p = exp2f(fmaf(s, scale_log2, -L2));
            pdp = p * dp;
        }
        Dacc += pdp;
        Pacc += p;
        for (int j = 0; j < kKeyTile; ++j) {
            const float pj = __shfl_sync(0xffffffffu, p, j);
            const float pdpj = __shfl_sync(0xffffffffu, pdp, j);
#pragma unroll
            for (int r = 0; r < PER_LANE; ++r) {
                const float kx = Ks[j][lane + 32 * r];
                ga[r] = fmaf(pdpj, kx, ga[r]);
                gb[r] = fmaf(pj, kx, gb[r]);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        Dacc += __shfl_xor_sync(0xffffffffu, Dacc, off);
        Pacc += __shfl_xor_sync(0xffffffffu, Pacc, off);
    }
    Dacc = row_ok ? Dacc / Pacc : 0.f;  // every valid row sees at least one key
    if (row_ok) {
#pragma unroll
        for (int r = 0; r < PER_LANE; ++r) dq[qrow * D + lane + 32 * r] = (ga[r] - Dacc * gb[r]) * scale;
        if (lane == 0) {
            const size_t ro = bg * rows_pad + (size_t)(h % G) * T + i;
            Drow[ro] = Dacc;
            L2row[ro] = L2;
        }
    }
}

constexpr int kKeysPerBlock = 8;   // dk, dv: one warp per key
constexpr int kRowTile = 32;       // query rows staged per round

// dk and dv of kKeysPerBlock keys of one KV head: one warp per key, each lane
// holding d / 32 columns of the key's k, v, dk and dv; query rows of the
// group's heads staged in tiles of 32. Key index u < C is cache slot u
// (empty slots u >= n get zero gradients), u >= C is chunk token u - C.
template <typename E, int D>
__global__ void __launch_bounds__(kKeysPerBlock * 32)
bwd_dkdv_simt_kernel(const E* __restrict__ q, const E* __restrict__ Kc, const E* __restrict__ Vc,
                     const E* __restrict__ k, const E* __restrict__ v, const E* __restrict__ dout,
                     const float* __restrict__ Drow, const float* __restrict__ L2row, float* __restrict__ dKc,
                     float* __restrict__ dVc, float* __restrict__ dk, float* __restrict__ dv, int Hq, int Hkv,
                     int C, int T, int n, int rows_pad, float scale_log2, float scale) {
    __shared__ float Qs[kRowTile][D];
    __shared__ float Os[kRowTile][D];
    __shared__ float Ls[kRowTile], Ds[kRowTile];
    constexpr int PER_LANE = D / 32;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    const size_t bg = (size_t)b * Hkv + g;
    const int u0 = blockIdx.x * kKeysPerBlock;
    const int u = u0 + warp;
    const bool is_cache = u < C;
    const bool valid = is_cache ? u < n : u < C + T;
    const int t_self = u - C;  // chunk token index (negative for cache slots)
    float kr[PER_LANE], vr[PER_LANE], gk[PER_LANE], gv[PER_LANE];
#pragma unroll
    for (int r = 0; r < PER_LANE; ++r) {
        const int x = lane + 32 * r;
        kr[r] = vr[r] = gk[r] = gv[r] = 0.f;
        if (valid) {
            kr[r] = to_f32(is_cache ? Kc[(bg * C + u) * D + x] : k[(bg * T + t_self) * D + x]);
            vr[r] = to_f32(is_cache ? Vc[(bg * C + u) * D + x] : v[(bg * T + t_self) * D + x]);
        }
    }
    // the first row any key of the block is visible to: 0 for cache slots,
    // otherwise the first chunk token's own row
    const int first_row = u0 < C ? 0 : u0 - C;
    for (int hh = 0; hh < G; ++hh) {
        const size_t qh = (size_t)b * Hq + (size_t)g * G + hh;
        for (int i0 = first_row; i0 < T; i0 += kRowTile) {
            __syncthreads();
            for (int e = threadIdx.x; e < kRowTile * D; e += blockDim.x) {
                const int r = e / D, x = e % D, i = i0 + r;
                Qs[r][x] = i < T ? to_f32(q[(qh * T + i) * D + x]) : 0.f;
                Os[r][x] = i < T ? to_f32(dout[(qh * T + i) * D + x]) : 0.f;
            }
            if (threadIdx.x < kRowTile) {
                const int i = i0 + threadIdx.x;
                const size_t ro = bg * rows_pad + (size_t)hh * T + (i < T ? i : 0);
                Ls[threadIdx.x] = i < T ? L2row[ro] : 0.f;
                Ds[threadIdx.x] = i < T ? Drow[ro] : 0.f;
            }
            __syncthreads();
            if (!valid) continue;
            for (int r = 0; r < kRowTile; ++r) {
                const int i = i0 + r;
                if (i >= T || i < t_self) continue;  // the row does not see this key (warp-uniform)
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int c = 0; c < PER_LANE; ++c) {
                    s = fmaf(Qs[r][lane + 32 * c], kr[c], s);
                    dp = fmaf(Os[r][lane + 32 * c], vr[c], dp);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    s += __shfl_xor_sync(0xffffffffu, s, off);
                    dp += __shfl_xor_sync(0xffffffffu, dp, off);
                }
                const float p = exp2f(fmaf(s, scale_log2, -Ls[r]));
                const float ds = p * (dp - Ds[r]);
#pragma unroll
                for (int c = 0; c < PER_LANE; ++c) {
                    gv[c] = fmaf(p, Os[r][lane + 32 * c], gv[c]);
                    gk[c] = fmaf(ds, Qs[r][lane + 32 * c], gk[c]);
                }
            }
        }
    }
    if (u >= C + T) return;
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) {
        const int x = lane + 32 * c;
        if (is_cache) {
            dKc[(bg * C + u) * D + x] = gk[c] * scale;  // zero for empty slots
            dVc[(bg * C + u) * D + x] = gv[c];
        } else {
            dk[(bg * T + t_self) * D + x] = gk[c] * scale;
            dv[(bg * T + t_self) * D + x] = gv[c];
        }
    }
}

template <typename E, int D>
cudaError_t bwd_simt_typed(const BwdArgs& a) {
    const float scale = 1.f / sqrtf((float)D);
    const float scale_log2 = kLog2e * scale;
    dim3 gq((a.T + kRowsPerBlock - 1) / kRowsPerBlock, a.Hq, a.B);
    bwd_dq_simt_kernel<E, D><<<gq, kRowsPerBlock * 32, 0, a.stream>>>(
        (const E*)a.q, (const E*)a.Kc, (const E*)a.Vc, (const E*)a.k, (const E*)a.v, (const E*)a.dout, a.lse,
        a.Drow, a.L2row, a.dq, a.Hq, a.Hkv, a.C, a.T, a.n, a.rows_pad, scale_log2, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    a.log->done("bwd_dq_simt_kernel", a.stream);
    dim3 gk((a.C + a.T + kKeysPerBlock - 1) / kKeysPerBlock, a.Hkv, a.B);
    bwd_dkdv_simt_kernel<E, D><<<gk, kKeysPerBlock * 32, 0, a.stream>>>(
        (const E*)a.q, (const E*)a.Kc, (const E*)a.Vc, (const E*)a.k, (const E*)a.v, (const E*)a.dout, a.Drow,
        a.L2row, a.dKc, a.dVc, a.dk, a.dv, a.Hq, a.Hkv, a.C, a.T, a.n, a.rows_pad, scale_log2, scale);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    a.log->done("bwd_dkdv_simt_kernel", a.stream);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_bwd_simt(const BwdArgs& a) {
    if (a.dtype == 1) return a.d == 64 ? bwd_simt_typed<float, 64>(a) : bwd_simt_typed<float, 128>(a);
    return a.d == 64 ? bwd_simt_typed<__nv_bfloat16, 64>(a) : bwd_simt_typed<__nv_bfloat16, 128>(a);
}

}  // namespace h2o
