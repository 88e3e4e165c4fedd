// decode.cu -- the H2O step for short chunks (decode: T <= kDecodeMaxT new
// tokens per sequence), same results as the chunk path, different schedule.
//
// With few query rows per KV group (R = G * T <= kDecodeMaxRows) the step is bound by
// reading the cache, not by arithmetic, so it is split over the keys
// ("split-K") instead of over query rows:
//   decode_split_kernel    one CTA per (KV group, slice of kDecodeSplit cache
//                          slots; one more slice holds the chunk's T tokens):
//                          scaled logits of all R rows against the slice,
//                          per-row partial softmax (max, sum, unnormalised
//                          P V), and the logits kept for the weight sums;
//   decode_combine_kernel  one CTA per query row: merges the slices into O
//                          and the row's log-sum-exp;
//   decode_wsum_kernel     one thread per candidate key: the summed attention
//                          weight exp(l - LSE) over the group's rows that see
//                          it, from the kept logits (no second Q K^T).
// The selection and copy kernels of the chunk path then run unchanged.
//
// What the step computes: "Learning how to Forget", paper page, section
// "Kernel Support Needs" (SDPA under the positional mask, summed weights per
// key) and section "Improvements to Heavy-Hitter Oracle (H2O)" (scores).
#include "kernels.h"

namespace h2o {
namespace {

constexpr int kDecThreads = 256;

template <int D>
struct DecSmem {
    // Q [R][D], K slice [S][D + 1] (padded: consecutive keys in consecutive
    // banks), V slice [S][D], logits / weights [R][S]; all fp32
    static size_t bytes(int R) {
        return sizeof(float) * ((size_t)R * D + (size_t)kDecodeSplit * (D + 1) + (size_t)kDecodeSplit * D +
                                (size_t)R * kDecodeSplit);
    }
};

template <typename E, int D>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const E* __restrict__ q, const E* __restrict__ k, const E* __restrict__ v,
                    const E* __restrict__ Kc, const E* __restrict__ Vc, float* __restrict__ part,
                    float* __restrict__ logits, int Hq, int Hkv, int C, int T, int n, int nsplit,
                    int lstride, float scale_log2) {
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ float dsm[];
    const int G = Hq / Hkv, R = G * T;
    const int s = blockIdx.x, bg = blockIdx.y;
    const int b = bg / Hkv, g = bg % Hkv;
    const int nsc = nsplit - 1;               // cache slices; slice nsc is the chunk
    const bool chunk = s == nsc;
    const int j0 = chunk ? 0 : s * kDecodeSplit;
    const int nk = chunk ? T : min(kDecodeSplit, n - j0);
    float* Qs = dsm;                          // [R][D]
    float* Ks = Qs + (size_t)R * D;           // [kDecodeSplit][D + 1]
    float* Vs = Ks + (size_t)kDecodeSplit * (D + 1);
    float* Ss = Vs + (size_t)kDecodeSplit * D;  // [R][kDecodeSplit]

    // stage Q rows (r = head-in-group * T + i) and the slice's K and V rows
    for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
        const int r = e / D, x = e % D;
        const int h = g * G + r / T, i = r % T;
        Qs[e] = to_f32(q[(((size_t)b * Hq + h) * T + i) * D + x]);
    }
    const E* ksrc = chunk ? k + (size_t)bg * T * D : Kc + ((size_t)bg * C + j0) * D;
    const E* vsrc = chunk ? v + (size_t)bg * T * D : Vc + ((size_t)bg * C + j0) * D;
    constexpr int V16 = 16 / (int)sizeof(E);  // elements per 16-byte load (rows are 16-byte aligned)
#pragma unroll 4
    for (int e = threadIdx.x * V16; e < nk * D; e += blockDim.x * V16) {
        const int j = e / D, x = e % D;
        E kv[V16], vv[V16];
        *reinterpret_cast<uint4*>(kv) = *reinterpret_cast<const uint4*>(ksrc + e);
        *reinterpret_cast<uint4*>(vv) = *reinterpret_cast<const uint4*>(vsrc + e);
#pragma unroll
        for (int u = 0; u < V16; ++u) {
            Ks[j * (D + 1) + x + u] = to_f32(kv[u]);
            Vs[e + u] = to_f32(vv[u]);
        }
    }
    __syncthreads();

    // scaled logits (log2 domain); chunk key t is visible to row i iff t <= i
    for (int e = threadIdx.x; e < R * nk; e += blockDim.x) {
        const int r = e / nk, j = e % nk;
        const float* qr = Qs + (size_t)r * D;
        const float* kj = Ks + (size_t)j * (D + 1);
        float acc = 0.f;
#pragma unroll 8
        for (int x = 0; x < D; ++x) acc = fmaf(qr[x], kj[x], acc);
        float l = acc * scale_log2;
        if (chunk && j > r % T) l = -INFINITY;
        Ss[(size_t)r * kDecodeSplit + j] = l;
        logits[((size_t)bg * R + r) * lstride + (chunk ? n + j : j0 + j)] = l;
    }
    __syncthreads();

    // per row: maximum, then weights 2^(l - m) in place and their sum
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
    for (int r = warp; r < R; r += nwarps) {
        float* Sr = Ss + (size_t)r * kDecodeSplit;
        float m = -INFINITY;
        for (int j = lane; j < nk; j += 32) m = fmaxf(m, Sr[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
        for (int j = lane; j < nk; j += 32) {
            const float p = (m == -INFINITY) ? 0.f : exp2f(Sr[j] - m);
            Sr[j] = p;
            l += p;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            float* pr = part + (((size_t)bg * nsplit + s) * R + r) * (D + 2);
            pr[D] = m;
            pr[D + 1] = l;
        }
    }
    __syncthreads();

    // unnormalised partial output P V of every row
    for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
        const int r = e / D, x = e % D;
        const float* Pr = Ss + (size_t)r * kDecodeSplit;
        float acc = 0.f;
        for (int j = 0; j < nk; ++j) acc = fmaf(Pr[j], Vs[(size_t)j * D + x], acc);
        part[(((size_t)bg * nsplit + s) * R + r) * (D + 2) + x] = acc;
    }
}

// One CTA per (query row r, group): O = sum_s 2^(m_s - M) O_s / L and the
// row's log-sum-exp, with M = max_s m_s, L = sum_s 2^(m_s - M) l_s (slices
// with no visible key have m_s = -inf and add nothing). Four groups of D
// threads each merge every fourth slice online (thread x holds column x),
// twelve slices' loads in flight at a time, and the four results meet in
// shared memory: a long chain of dependent loads would bound this kernel.
constexpr int kCombGroups = 4;
constexpr int kCombBatch = 12;

template <typename E, int D>
__global__ void __launch_bounds__(kCombGroups * D)
decode_combine_kernel(const float* __restrict__ part, E* __restrict__ out, float* __restrict__ lse,
                      float* __restrict__ lse2_rows, int Hq, int Hkv, int T, int nsplit, int tmax) {
    griddep_wait();
    griddep_launch_dependents();
    const int G = Hq / Hkv, R = G * T;
    const int r = blockIdx.x, bg = blockIdx.y;
    const int b = bg / Hkv, g = bg % Hkv;
    const int h = g * G + r / T, i = r % T;
    const float* pr = part + ((size_t)bg * nsplit * R + r) * (D + 2);
    const size_t sstride = (size_t)R * (D + 2);
    const int x = threadIdx.x % D, sg = threadIdx.x / D;
    float M = -INFINITY, L = 0.f, acc = 0.f;
    for (int s0 = sg; s0 < nsplit; s0 += kCombGroups * kCombBatch) {
        float ms[kCombBatch], ls[kCombBatch], os[kCombBatch];
#pragma unroll
        for (int u = 0; u < kCombBatch; ++u) {
            const int sl = s0 + kCombGroups * u;
            const bool on = sl < nsplit;
            ms[u] = on ? pr[sl * sstride + D] : -INFINITY;
            ls[u] = on ? pr[sl * sstride + D + 1] : 0.f;
            os[u] = on ? pr[sl * sstride + x] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kCombBatch; ++u) {
            if (ms[u] == -INFINITY) continue;
            const float Mn = fmaxf(M, ms[u]);
            const float a = exp2f(M - Mn);  // 0 while M is -inf
            const float w = exp2f(ms[u] - Mn);
            acc = fmaf(acc, a, w * os[u]);
            L = fmaf(L, a, w * ls[u]);
            M = Mn;
        }
    }
    __shared__ float gM[kCombGroups], gL[kCombGroups];
    __shared__ float gacc[kCombGroups][D];
    gacc[sg][x] = acc;
    if (x == 0) {
        gM[sg] = M;
        gL[sg] = L;
    }
    __syncthreads();
    if (sg != 0) return;
    float Mt = gM[0];
#pragma unroll
    for (int q2 = 1; q2 < kCombGroups; ++q2) Mt = fmaxf(Mt, gM[q2]);
    float Lt = 0.f, at = 0.f;
#pragma unroll
    for (int q2 = 0; q2 < kCombGroups; ++q2) {
        const float w = gM[q2] == -INFINITY ? 0.f : exp2f(gM[q2] - Mt);
        Lt = fmaf(w, gL[q2], Lt);
        at = fmaf(w, gacc[q2][x], at);
    }
    out[(((size_t)b * Hq + h) * T + i) * D + x] = from_f32<E>(at / Lt);
    if (x == 0) {
        const float l2 = Mt + log2f(Lt);
        lse[((size_t)b * Hq + h) * tmax + i] = l2 * kLn2;
        lse2_rows[(size_t)bg * R + r] = l2;
    }
}

// One thread per candidate c of a group (cache slots 0..n-1, then chunk
// tokens n..n+T-1): the weight it receives, summed over the group's rows in
// row order; masked pairs hold -inf logits and add 0.
__global__ void __launch_bounds__(kDecThreads)
decode_wsum_kernel(const float* __restrict__ logits, const float* __restrict__ lse2_rows,
                   float* __restrict__ partials, int R, int n, int T, int lstride, int cstride) {
    griddep_wait();
    griddep_launch_dependents();
    const int bg = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= n + T) return;
    const float* lr = logits + (size_t)bg * R * lstride + c;
    const float* l2 = lse2_rows + (size_t)bg * R;
    float acc = 0.f;
#pragma unroll 8
    for (int r = 0; r < R; ++r) acc += exp2f(lr[(size_t)r * lstride] - l2[r]);
    partials[(size_t)bg * cstride + c] = acc;
}

template <typename E, int D>
cudaError_t launch_decode_typed(const StepArgs& a) {
    const int G = a.Hq / a.Hkv, R = G * a.T, groups = a.B * a.Hkv;
    const int nsplit = (a.n + kDecodeSplit - 1) / kDecodeSplit + 1;
    const int lstride = a.C + kDecodeMaxT;
    const size_t smem = DecSmem<D>::bytes(R);
    if (cudaError_t e = ensure_smem_limit(decode_split_kernel<E, D>, (int)DecSmem<D>::bytes(kDecodeMaxRows));
        e != cudaSuccess)
        return e;
    const float scale_log2 = kLog2e / sqrtf((float)D);
    cudaError_t e = launch_ex(true, decode_split_kernel<E, D>, dim3(nsplit, groups), dim3(kDecThreads), smem,
                              a.stream, (const E*)a.q, (const E*)a.k, (const E*)a.v, (const E*)a.Kc,
                              (const E*)a.Vc, a.dec_part, a.dec_logits, a.Hq, a.Hkv, a.C, a.T, a.n, nsplit,
                              lstride, scale_log2);
    if (e != cudaSuccess) return e;
    a.log->done("decode_split_kernel", a.stream);
    e = launch_ex(true, decode_combine_kernel<E, D>, dim3(R, groups), dim3(kCombGroups * D), 0, a.stream,
                  (const float*)a.dec_part, (E*)a.out, a.lse, a.dec_lse2, a.Hq, a.Hkv, a.T, nsplit, a.tmax);
    if (e != cudaSuccess) return e;
    a.log->done("decode_combine_kernel", a.stream);
    e = launch_ex(true, decode_wsum_kernel, dim3((a.n + a.T + kDecThreads - 1) / kDecThreads, groups),
                  dim3(kDecThreads), 0, a.stream, (const float*)a.dec_logits, (const float*)a.dec_lse2,
                  a.partials, R, a.n, a.T, lstride, cand_stride(a));
    if (e != cudaSuccess) return e;
    a.log->done("decode_wsum_kernel", a.stream);
    return cudaGetLastError();
}

}  // namespace

bool decode_applies(int Hq, int Hkv, int d, int T) {
    return T <= kDecodeMaxT && (Hq / Hkv) * T <= kDecodeMaxRows && (d == 64 || d == 128);
}

size_t decode_part_floats(int B, int Hq, int Hkv, int d, int C) {
    const int nsplit = (C + kDecodeSplit - 1) / kDecodeSplit + 1;
    return (size_t)B * Hkv * nsplit * kDecodeMaxRows * (d + 2);
}

size_t decode_logit_floats(int B, int Hkv, int C) { return (size_t)B * Hkv * kDecodeMaxRows * (C + kDecodeMaxT); }

size_t decode_lse2_floats(int B, int Hkv) { return (size_t)B * Hkv * kDecodeMaxRows; }

cudaError_t launch_decode(const StepArgs& a) {
    if (a.dtype == 1) return a.d == 64 ? launch_decode_typed<float, 64>(a) : launch_decode_typed<float, 128>(a);
    return a.d == 64 ? launch_decode_typed<__nv_bfloat16, 64>(a) : launch_decode_typed<__nv_bfloat16, 128>(a);
}

}  // namespace h2o
