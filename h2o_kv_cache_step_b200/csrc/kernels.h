// kernels.h -- internal launch interface of the H2O step kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"

namespace h2o {

// Names (and, when profiling, events) of the kernels one step launches.
// Every launcher calls done() right after each of its launches.
constexpr int kMaxStepKernels = 8;
struct LaunchLog {
    cudaEvent_t* ev = nullptr;   // kMaxStepKernels + 1 events, or nullptr
    const char* names[kMaxStepKernels];
    int n = 0;
    void done(const char* name, cudaStream_t s) {
        if (n >= kMaxStepKernels) return;
        names[n++] = name;
        if (ev) cudaEventRecord(ev[n], s);
    }
};

// Everything one step's kernels read or write. Device pointers unless noted.
struct StepArgs {
    int B, Hq, Hkv, d, C, T;
    int n;            // valid cache slots (prefix 0..n-1) before the step
    int64_t P;        // position of the chunk's first token
    int dtype;        // 0 = bf16, 1 = fp32
    int policy;       // eviction ranking: 0 = H2O score, 1 = score / age
    int tmax;         // capacity (in tokens) of the per-step workspace
    int early;        // the previous kernel on the stream is this context's
                      // own step: the SDPA may attend to the chunk's keys
                      // before that step has finished (tensor-core path)
    const void* q;    // [B,Hq,T,d]
    const void* k;    // [B,Hkv,T,d]
    const void* v;    // [B,Hkv,T,d]
    void* out;        // [B,Hq,T,d]
    void* Kc;         // [B,Hkv,C,d] cache keys
    void* Vc;         // [B,Hkv,C,d] cache values
    float* scores;    // [B,Hkv,C]
    int32_t* pos;     // [B,Hkv,C]
    float* lse;       // [B,Hq,tmax] natural-log normaliser per row
    float* nlse2;     // [B*Hkv, rows_pad] -log2 normaliser per flattened group row (tensor-core path)
    int rows_pad;
    float* cand_score;   // [B,Hkv,C+tmax]
    int32_t* cand_pos;   // [B,Hkv,C+tmax]
    uint8_t* cand_kept;  // [B,Hkv,C+tmax]
    int32_t* token_slot; // [B,Hkv,tmax]
    float* partials;     // weight-sum partials [nparts][B*Hkv][C+tmax] (tensor-core path)
    size_t partial_elems;
    int nparts;          // > 0: the selection kernel first sums the partials
    void* ins_K;         // insert-always: compact K of the kept entries [B,Hkv,C,d]
    void* ins_V;         // insert-always: compact V
    int32_t* ins_slot;   // insert-always: slot of compact entry r [B*Hkv][C]
    float* ins_score;    // insert-always: its score before the step
    int32_t* ins_pos;    // insert-always: its position
    float* dec_part;     // decode path: per-(group, slice, row) partial O, max, sum
    float* dec_logits;   // decode path: scaled logits [group][row][C + kDecodeMaxT]
    float* dec_lse2;     // decode path: log2-sum-exp per (group, row)
    const void* tmaps;   // device copy of the step's TMA descriptors (tensor-core path)
    float* sdpa_part;    // split SDPA: partial outputs, maxima and sums (tensor-core path)
    size_t sdpa_part_elems;
    WaitBound wb;
    cudaStream_t stream;
    int num_sms;
    LaunchLog* log;
};

inline int cand_stride(const StepArgs& a) { return a.C + a.tmax; }

// Launch `kernel` on `stream`, allowing programmatic dependent launch if `pdl`
// (every kernel calls griddep_wait() before it touches global memory that
// earlier work writes, so both modes are correct).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// As launch_ex, with programmatic dependent launch only if H2O_PDL is defined.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
#ifdef H2O_PDL
    const bool pdl = true;
#else
    const bool pdl = false;  // measured: no gain for the tensor-core kernels
#endif
    return launch_ex(pdl, kernel, grid, block, smem, stream, args...);
}

// Raise `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel, device); safe to call from several threads.
template <typename... KArgs>
cudaError_t ensure_smem_limit(void (*kernel)(KArgs...), int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    const std::pair<const void*, int> key(reinterpret_cast<const void*>(kernel), dev);
    std::lock_guard<std::mutex> lock(mu);
    if (done.count(key)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert(key);
    return e;
}

// SIMT kernels (fp32 path; any supported d).
cudaError_t launch_sdpa_simt(const StepArgs& a);
cudaError_t launch_wsum_simt(const StepArgs& a);
// Eviction: per (sequence, KV head) radix select + slot map + K/V copy.
// Decode path (short chunks): split-K SDPA, combine, weight sums from the
// kept logits; then launch_select with nparts = 1.
constexpr int kDecodeMaxT = 16;      // longest chunk the decode path takes
// query rows per KV group (G * T) it takes: the split kernel's dot products
// run on the CUDA cores, and above this the tensor-core chunk path is faster
// (measured: 64 rows, T = 16 at G = 4: 113 us per step here against 73)
constexpr int kDecodeMaxRows = 32;
constexpr int kDecodeSplit = 64;     // cache slots per split
bool decode_applies(int Hq, int Hkv, int d, int T);
size_t decode_part_floats(int B, int Hq, int Hkv, int d, int C);
size_t decode_logit_floats(int B, int Hkv, int C);
size_t decode_lse2_floats(int B, int Hkv);
cudaError_t launch_decode(const StepArgs& a);

// Insert-always variant: eviction before the attention, then the chunk step
// over the compact cache of the kept entries.
cudaError_t launch_insert_select(const StepArgs& a, int n_kept);
cudaError_t launch_gather(const StepArgs& a, int n_kept);
cudaError_t launch_insert_finish(const StepArgs& a, int n_kept);

// Backward of one step's chunk SDPA with the key set held fixed (the replay of
// a logged step): everything the kernels read or write. Device pointers.
struct BwdArgs {
    int B, Hq, Hkv, d, C, T;
    int n;              // valid cache slots (prefix 0..n-1) of the replayed pre-step cache
    int dtype;          // 0 = bf16, 1 = fp32 (inputs); gradients are fp32
    const void* q;      // [B,Hq,T,d]
    const void* k;      // [B,Hkv,T,d]
    const void* v;      // [B,Hkv,T,d]
    const float* lse;   // forward natural-log LSE [B,Hq,T]
    const void* dout;   // dL/dout [B,Hq,T,d]
    const void* Kc;     // [B,Hkv,C,d]
    const void* Vc;     // [B,Hkv,C,d]
    float* dq;          // [B,Hq,T,d]
    float* dKc;         // [B,Hkv,C,d] (zero in empty slots)
    float* dVc;         // [B,Hkv,C,d]
    float* dk;          // [B,Hkv,T,d]
    float* dv;          // [B,Hkv,T,d]
    float* Drow;        // [B*Hkv][rows_pad]: sum_j p_j dp_j / sum_j p_j per flattened group row (head-in-group * T + i)
    float* L2row;       // [B*Hkv][rows_pad]: log2-domain LSE per flattened group row
    int rows_pad;
    WaitBound wb;
    cudaStream_t stream;
    int num_sms;
    LaunchLog* log;
};
cudaError_t launch_bwd_simt(const BwdArgs& a);

// Selection, slot map and the kept tokens' K/V copy (sum and normalized
// policies); scatter_kernel's wide copy (insert-always).
cudaError_t launch_select(const StepArgs& a);
cudaError_t launch_scatter(const StepArgs& a);
// Sets the message h2o_last_error(NULL) reports on this thread.
void set_thread_error_message(const char* msg);
// Self-test of the bounded wait.
cudaError_t launch_wait_selftest(const WaitBound& wb, cudaStream_t s);

}  // namespace h2o
