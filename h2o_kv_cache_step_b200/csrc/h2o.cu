// h2o.cu -- the C ABI of the chunked H2O step (declared in include/h2o.h).
//
// Owns the context: the cache (keys, values, H2O scores, positions) for every
// (sequence, KV head), the per-step workspace and the device error word; and
// issues one step as a fixed, stream-ordered sequence of kernels:
//   1. chunk SDPA, writing the output and each row's log-sum-exp;
//   2. per-key attention-weight sums, added to the H2O scores;
//   3. selection of the C survivors and the token -> slot map;
//   4. copy of the surviving chunk keys/values into their slots.
// No step of the path runs on the host: the host validates arguments, keeps
// the two counters (P, n) and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/h2o.h"
#include "kernels.h"
#include "tc.h"

using namespace h2o;

namespace {

thread_local char g_thread_err[512] = "";

}  // namespace

void h2o::set_thread_error_message(const char* msg) {
    snprintf(g_thread_err, sizeof(g_thread_err), "%s", msg);
}

struct h2o_ctx {
    int B, Hq, Hkv, d, C, dtype, tmax;
    int policy = 0;  // H2O_POLICY_SUM
    int device;
    int num_sms;
    int64_t P, n;
    size_t elem;
    // cache
    void* Kc = nullptr;
    void* Vc = nullptr;
    float* scores = nullptr;
    int32_t* pos = nullptr;
    // workspace (capacity tmax tokens)
    float* lse = nullptr;
    float* cand_score = nullptr;
    int32_t* cand_pos = nullptr;
    uint8_t* cand_kept = nullptr;
    int32_t* token_slot = nullptr;
    float* partials = nullptr;
    size_t partial_elems = 0;
    float* nlse2 = nullptr;
    int rows_pad = 0;
    // insert-always workspace (allocated when the policy is first selected):
    // compact K/V of the kept entries, their slots, scores and positions
    void* ins_K = nullptr;
    void* ins_V = nullptr;
    int32_t* ins_slot = nullptr;
    float* ins_score = nullptr;
    int32_t* ins_pos = nullptr;
    // backward workspace (allocated on the first h2o_backward): dO . O and the
    // log2-domain LSE per flattened group row, [2][groups][bwd_rows_pad]
    float* bwd_rows = nullptr;
    int bwd_rows_pad = 0;
    // split SDPA workspace (grown on demand when a step splits its units)
    float* sdpa_part = nullptr;
    size_t sdpa_part_elems = 0;
    // decode-path workspace (chunks of up to kDecodeMaxT tokens)
    float* dec_part = nullptr;
    float* dec_logits = nullptr;
    float* dec_lse2 = nullptr;
    // host staging for h2o_step_host
    void* stage = nullptr;
    size_t stage_bytes = 0;
    // pipelined host path (h2o_step_host_async): two staging slots, an upload
    // and a download stream, and per-slot events
    void* aslot[2] = {nullptr, nullptr};
    size_t aslot_bytes = 0;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_in[2] = {nullptr, nullptr};    // slot's inputs uploaded
    cudaEvent_t ev_step[2] = {nullptr, nullptr};  // step reading the slot done
    cudaEvent_t ev_out[2] = {nullptr, nullptr};   // slot's output downloaded
    long long achunks = 0;
    // error word (host-mapped)
    int* err_host = nullptr;
    int* err_dev = nullptr;
    unsigned long long wait_ns;
    int poisoned = 0;
    // last step
    int last_T = 0, last_n = 0;
    bool use_tc = false;
    // per-kernel profiling
    bool prof_on = false;
    int prof_max_steps = 0, prof_steps = 0;
    std::vector<cudaEvent_t> prof_ev;      // (kMaxStepKernels + 1) per step
    std::vector<LaunchLog> prof_logs;
    char err[512];
};

namespace {

int fail(h2o_ctx* c, int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    if (c) {
        snprintf(c->err, sizeof(c->err), "%s", buf);
    } else {
        snprintf(g_thread_err, sizeof(g_thread_err), "%s", buf);
    }
    return code;
}

int cuda_fail(h2o_ctx* c, cudaError_t e, const char* what) {
    return fail(c, e == cudaErrorMemoryAllocation ? H2O_ERR_OOM : H2O_ERR_CUDA, "%s: %s (%s)", what,
                cudaGetErrorString(e), cudaGetErrorName(e));
}

#define H2O_TRY(ctx, expr, what)                        \
    do {                                                \
        cudaError_t e_ = (expr);                        \
        if (e_ != cudaSuccess) return cuda_fail(ctx, e_, what); \
    } while (0)

// Makes the context's device current for the lifetime of the object.
struct DeviceGuard {
    int prev = -1;
    bool changed = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
            changed = cudaSetDevice(dev) == cudaSuccess;
        }
    }
    ~DeviceGuard() {
        if (changed) cudaSetDevice(prev);
    }
};

// Releases the pipelined host path's streams, events and staging slots.
void free_async(h2o_ctx* c) {
    if (c->s_in) cudaStreamSynchronize(c->s_in);
    if (c->s_out) cudaStreamSynchronize(c->s_out);
    for (int i = 0; i < 2; ++i) {
        cudaFree(c->aslot[i]);
        c->aslot[i] = nullptr;
        for (cudaEvent_t* e : {&c->ev_in[i], &c->ev_step[i], &c->ev_out[i]}) {
            if (*e) cudaEventDestroy(*e);
            *e = nullptr;
        }
    }
    if (c->s_in) cudaStreamDestroy(c->s_in);
    if (c->s_out) cudaStreamDestroy(c->s_out);
    c->s_in = c->s_out = nullptr;
    c->aslot_bytes = 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void free_workspace(h2o_ctx* c) {
    cudaFree(c->lse);
    cudaFree(c->cand_score);
    cudaFree(c->cand_pos);
    cudaFree(c->cand_kept);
    cudaFree(c->token_slot);
    cudaFree(c->partials);
    cudaFree(c->nlse2);
    cudaFree(c->dec_part);
    cudaFree(c->dec_logits);
    cudaFree(c->dec_lse2);
    c->dec_part = c->dec_logits = c->dec_lse2 = nullptr;
    c->nlse2 = nullptr;
    c->lse = c->cand_score = c->partials = nullptr;
    c->cand_pos = c->token_slot = nullptr;
    c->cand_kept = nullptr;
    c->partial_elems = 0;
}

int alloc_workspace(h2o_ctx* c, int tmax) {
    const size_t groups = (size_t)c->B * c->Hkv;
    const size_t cs = (size_t)c->C + tmax;
    H2O_TRY(c, cudaMalloc(&c->lse, sizeof(float) * (size_t)c->B * c->Hq * tmax), "cudaMalloc(lse)");
    H2O_TRY(c, cudaMalloc(&c->cand_score, sizeof(float) * groups * cs), "cudaMalloc(cand_score)");
    H2O_TRY(c, cudaMalloc(&c->cand_pos, sizeof(int32_t) * groups * cs), "cudaMalloc(cand_pos)");
    H2O_TRY(c, cudaMalloc(&c->cand_kept, groups * cs), "cudaMalloc(cand_kept)");
    H2O_TRY(c, cudaMalloc(&c->token_slot, sizeof(int32_t) * groups * tmax), "cudaMalloc(token_slot)");
    c->partial_elems = tc_partial_elems(c->B, c->Hq, c->Hkv, c->C, tmax);
    if (c->partial_elems)
        H2O_TRY(c, cudaMalloc(&c->partials, sizeof(float) * c->partial_elems), "cudaMalloc(partials)");
    c->rows_pad = tc_rows_pad(c->Hq, c->Hkv, tmax);
    H2O_TRY(c, cudaMalloc(&c->nlse2, sizeof(float) * groups * (size_t)c->rows_pad), "cudaMalloc(nlse2)");
    if (decode_applies(c->Hq, c->Hkv, c->d, 1)) {
        H2O_TRY(c, cudaMalloc(&c->dec_part, sizeof(float) * decode_part_floats(c->B, c->Hq, c->Hkv, c->d, c->C)),
                "cudaMalloc(decode partials)");
        H2O_TRY(c, cudaMalloc(&c->dec_logits, sizeof(float) * decode_logit_floats(c->B, c->Hkv, c->C)),
                "cudaMalloc(decode logits)");
        H2O_TRY(c, cudaMalloc(&c->dec_lse2, sizeof(float) * decode_lse2_floats(c->B, c->Hkv)),
                "cudaMalloc(decode lse)");
    }
    c->tmax = tmax;
    return H2O_OK;
}

int check_ctx(h2o_ctx* c) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    if (c->poisoned) return fail(c, H2O_ERR_POISONED, "context poisoned by an earlier device error");
    const int word = *(volatile int*)c->err_host;
    if (word != kDevOk) {
        c->poisoned = 1;
        return fail(c, H2O_ERR_TIMEOUT, "a kernel stopped after a bounded wait ran out (device code %d)",
                    word);
    }
    return H2O_OK;
}

StepArgs make_args(h2o_ctx* c, const void* q, const void* k, const void* v, void* out, int T,
                   cudaStream_t s) {
    StepArgs a{};
    a.B = c->B;
    a.Hq = c->Hq;
    a.Hkv = c->Hkv;
    a.d = c->d;
    a.C = c->C;
    a.T = T;
    a.n = (int)c->n;
    a.P = c->P;
    a.dtype = c->dtype;
    a.policy = c->policy;
    a.tmax = c->tmax;
    a.q = q;
    a.k = k;
    a.v = v;
    a.out = out;
    a.Kc = c->Kc;
    a.Vc = c->Vc;
    a.scores = c->scores;
    a.pos = c->pos;
    a.lse = c->lse;
    a.cand_score = c->cand_score;
    a.cand_pos = c->cand_pos;
    a.cand_kept = c->cand_kept;
    a.token_slot = c->token_slot;
    a.partials = c->partials;
    a.partial_elems = c->partial_elems;
    a.nlse2 = c->nlse2;
    a.ins_K = c->ins_K;
    a.ins_V = c->ins_V;
    a.ins_slot = c->ins_slot;
    a.ins_score = c->ins_score;
    a.ins_pos = c->ins_pos;
    a.dec_part = c->dec_part;
    a.dec_logits = c->dec_logits;
    a.dec_lse2 = c->dec_lse2;
    a.rows_pad = c->rows_pad;
    a.wb.err_word = c->err_dev;
    a.wb.ns = c->wait_ns;
    a.stream = s;
    a.num_sms = c->num_sms;
    return a;
}

}  // namespace

extern "C" {

const char* h2o_version(void) { return "h2o_kv_cache_step_b200 0.1 (sm_100a)"; }

const char* h2o_last_error(const h2o_ctx* c) { return c ? c->err : g_thread_err; }

int h2o_create_ex(int B, int Hq, int Hkv, int d, int C, int dtype, int max_T, h2o_ctx** out) {
    if (!out) return fail(nullptr, H2O_ERR_ARG, "out is NULL");
    *out = nullptr;
    if (B < 1 || Hq < 1 || Hkv < 1 || C < 1 || max_T < 1)
        return fail(nullptr, H2O_ERR_ARG, "B, Hq, Hkv, C, max_T must be >= 1");
    if (Hq % Hkv != 0) return fail(nullptr, H2O_ERR_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (d != 64 && d != 128) return fail(nullptr, H2O_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
    if (dtype != H2O_BF16 && dtype != H2O_FP32) return fail(nullptr, H2O_ERR_ARG, "unknown dtype %d", dtype);
    if ((long long)C + max_T > (1ll << 30)) return fail(nullptr, H2O_ERR_UNSUPPORTED, "C + max_T too large");

    h2o_ctx* c = new (std::nothrow) h2o_ctx();
    if (!c) return fail(nullptr, H2O_ERR_OOM, "host allocation failed");
    c->B = B;
    c->Hq = Hq;
    c->Hkv = Hkv;
    c->d = d;
    c->C = C;
    c->dtype = dtype;
    c->elem = dtype == H2O_FP32 ? 4 : 2;
    c->P = 0;
    c->n = 0;
    c->err[0] = 0;
    const char* env = getenv("H2O_WAIT_TIMEOUT_MS");
    long long ms = env ? atoll(env) : 0;
    c->wait_ns = (unsigned long long)(ms > 0 ? ms : 2000) * 1000000ull;

    auto bail = [&](int rc) {
        snprintf(g_thread_err, sizeof(g_thread_err), "%s", c->err);
        h2o_destroy(c);
        return rc;
    };
    cudaError_t e = cudaGetDevice(&c->device);
    if (e != cudaSuccess) return bail(cuda_fail(c, e, "cudaGetDevice"));
    e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
    if (e != cudaSuccess) return bail(cuda_fail(c, e, "cudaDeviceGetAttribute"));
    const size_t groups = (size_t)B * Hkv;
    const size_t cache_bytes = groups * C * d * c->elem;
    if ((e = cudaMalloc(&c->Kc, cache_bytes)) != cudaSuccess) return bail(cuda_fail(c, e, "cudaMalloc(K cache)"));
    if ((e = cudaMalloc(&c->Vc, cache_bytes)) != cudaSuccess) return bail(cuda_fail(c, e, "cudaMalloc(V cache)"));
    if ((e = cudaMalloc(&c->scores, sizeof(float) * groups * C)) != cudaSuccess)
        return bail(cuda_fail(c, e, "cudaMalloc(scores)"));
    if ((e = cudaMalloc(&c->pos, sizeof(int32_t) * groups * C)) != cudaSuccess)
        return bail(cuda_fail(c, e, "cudaMalloc(positions)"));
    int rc = alloc_workspace(c, max_T);
    if (rc != H2O_OK) return bail(rc);
    if ((e = cudaHostAlloc((void**)&c->err_host, sizeof(int), cudaHostAllocMapped)) != cudaSuccess)
        return bail(cuda_fail(c, e, "cudaHostAlloc(error word)"));
    *c->err_host = kDevOk;
    if ((e = cudaHostGetDevicePointer((void**)&c->err_dev, c->err_host, 0)) != cudaSuccess)
        return bail(cuda_fail(c, e, "cudaHostGetDevicePointer(error word)"));
    c->use_tc = (dtype == H2O_BF16) && tc_supported(c->device, d);
    rc = h2o_reset(c, nullptr);
    if (rc != H2O_OK) return bail(rc);
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return bail(cuda_fail(c, e, "initial clear"));
    *out = c;
    return H2O_OK;
}

int h2o_create(int B, int Hq, int Hkv, int d, int C, h2o_ctx** out) {
    return h2o_create_ex(B, Hq, Hkv, d, C, H2O_BF16, C, out);
}

int h2o_destroy(h2o_ctx* c) {
    if (!c) return H2O_OK;
    DeviceGuard g(c->device);
    cudaDeviceSynchronize();
    free_async(c);
    free_workspace(c);
    for (cudaEvent_t e : c->prof_ev) cudaEventDestroy(e);
    cudaFree(c->Kc);
    cudaFree(c->Vc);
    cudaFree(c->bwd_rows);
    cudaFree(c->sdpa_part);
    cudaFree(c->ins_K);
    cudaFree(c->ins_V);
    cudaFree(c->ins_slot);
    cudaFree(c->ins_score);
    cudaFree(c->ins_pos);
    cudaFree(c->scores);
    cudaFree(c->pos);
    cudaFree(c->stage);
    if (c->err_host) cudaFreeHost(c->err_host);
    delete c;
    return H2O_OK;
}

int h2o_reset(h2o_ctx* c, void* stream) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t groups = (size_t)c->B * c->Hkv;
    H2O_TRY(c, cudaMemsetAsync(c->scores, 0, sizeof(float) * groups * c->C, s), "reset scores");
    H2O_TRY(c, cudaMemsetAsync(c->pos, 0xff, sizeof(int32_t) * groups * c->C, s), "reset positions");
    H2O_TRY(c, cudaMemsetAsync(c->Kc, 0, groups * c->C * c->d * c->elem, s), "reset K");
    H2O_TRY(c, cudaMemsetAsync(c->Vc, 0, groups * c->C * c->d * c->elem, s), "reset V");
    c->P = 0;
    c->n = 0;
    c->last_T = 0;
    c->last_n = 0;
    return H2O_OK;
}

int h2o_kernel_plan(const h2o_ctx* c, int T, const char** names, int max_names) {
    if (!c || T < 1) return fail(nullptr, H2O_ERR_ARG, "bad arguments");
    const char* plan[kMaxStepKernels];
    int k = 0;
    const bool insert = c->policy == H2O_POLICY_INSERT_ALWAYS;
    if (insert) {
        plan[k++] = "insert_select_kernel";
        plan[k++] = "gather_kernel";
    }
    if (c->dec_part && decode_applies(c->Hq, c->Hkv, c->d, T)) {
        plan[k++] = "decode_split_kernel";
        plan[k++] = "decode_combine_kernel";
        plan[k++] = "decode_wsum_kernel";
    } else if (c->use_tc) {
        const int n_eff = insert ? (int)(c->n + T > c->C ? c->C - T : c->n) : (int)c->n;
        k += tc_kernel_plan(c->B, c->Hq, c->Hkv, c->d, c->C, T, n_eff, c->num_sms, plan + k,
                            kMaxStepKernels - 2 - k);
    } else {
        plan[k++] = "sdpa_simt_kernel";
        plan[k++] = "wsum_simt_kernel";
    }
    plan[k++] = insert ? "insert_finish_kernel" : "select_kernel";
    if (insert) plan[k++] = "scatter_kernel";
    for (int i = 0; i < k && i < max_names; ++i)
        if (names) names[i] = plan[i];
    return k;
}

// One step. early: the previous kernel on the stream is this context's own
// previous step (h2o_prefill), so the tensor-core SDPA may attend to the
// chunk's own keys while that step's eviction still runs.
static int step_impl(h2o_ctx* c, const void* q, const void* k, const void* v, void* out, int T, void* stream,
                     bool early) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (T < 1) return fail(c, H2O_ERR_ARG, "T must be >= 1 (got %d)", T);
    if (!q || !k || !v || !out) return fail(c, H2O_ERR_ARG, "q, k, v, out must be non-NULL");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(c, H2O_ERR_ALIGN, "q, k, v, out must be 16-byte aligned");
    if (c->P + T > (int64_t)INT32_MAX) return fail(c, H2O_ERR_UNSUPPORTED, "positions would exceed 2^31-1");
    if (c->policy == H2O_POLICY_INSERT_ALWAYS && T > c->C)
        return fail(c, H2O_ERR_UNSUPPORTED, "insert-always needs T <= C (T = %d, C = %d)", T, c->C);
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    if (T > c->tmax) {
        H2O_TRY(c, cudaStreamSynchronize(s), "sync before workspace growth");
        H2O_TRY(c, cudaDeviceSynchronize(), "sync before workspace growth");
        free_workspace(c);
        rc = alloc_workspace(c, T);
        if (rc != H2O_OK) return rc;
    }
    StepArgs a = make_args(c, q, k, v, out, T, s);
    LaunchLog local_log;
    a.log = &local_log;
    if (c->prof_on && c->prof_steps < c->prof_max_steps) {
        const int slot = c->prof_steps++;
        a.log = &c->prof_logs[slot];
        a.log->n = 0;
        a.log->ev = &c->prof_ev[(size_t)slot * (kMaxStepKernels + 1)];
        H2O_TRY(c, cudaEventRecord(a.log->ev[0], s), "record profiling event");
    }
    const bool decode = c->dec_part && decode_applies(c->Hq, c->Hkv, c->d, T);
    a.nparts = decode ? 1 : c->use_tc ? tc_partial_count(c->Hq, c->Hkv, T) : 0;
    // insert-always: eviction first, then the chunk step over the compact
    // cache of the kept entries (attention and weight sums unchanged)
    const bool insert = c->policy == H2O_POLICY_INSERT_ALWAYS;
    // profiling puts events between the kernels, which ends the overlap
    a.early = early && !insert && !decode && c->use_tc && a.log == &local_log;
    const int n_kept = insert ? (int)(c->n + T > c->C ? c->C - T : c->n) : (int)c->n;
    StepArgs b = a;
    if (insert) {
        H2O_TRY(c, launch_insert_select(a, n_kept), "launch insert-always selection");
        H2O_TRY(c, launch_gather(a, n_kept), "launch gather of the kept entries");
        b.Kc = c->ins_K;
        b.Vc = c->ins_V;
        b.n = n_kept;
        b.scores = c->ins_score;
        b.pos = c->ins_pos;
    }
    if (decode) {
        H2O_TRY(c, launch_decode(b), "launch decode-path kernels");
    } else if (c->use_tc) {
        const size_t need = tc_sdpa_part_elems(c->B, c->Hq, c->Hkv, c->d, T, (int)b.n, c->num_sms);
        if (need > c->sdpa_part_elems) {
            // the first split step, or one that needs more room: (re)allocate once
            if (c->sdpa_part) {
                H2O_TRY(c, cudaStreamSynchronize(s), "sync before SDPA workspace growth");
                H2O_TRY(c, cudaDeviceSynchronize(), "sync before SDPA workspace growth");
                cudaFree(c->sdpa_part);
                c->sdpa_part = nullptr;
                c->sdpa_part_elems = 0;
            }
            H2O_TRY(c, cudaMalloc(&c->sdpa_part, sizeof(float) * need), "cudaMalloc(split SDPA workspace)");
            c->sdpa_part_elems = need;
        }
        b.sdpa_part = c->sdpa_part;
        b.sdpa_part_elems = c->sdpa_part_elems;
        H2O_TRY(c, tc_sdpa(b), "launch tensor-core SDPA");
        H2O_TRY(c, tc_wsum(b), "launch tensor-core weight sums");
    } else {
        H2O_TRY(c, launch_sdpa_simt(b), "launch SDPA");
        H2O_TRY(c, launch_wsum_simt(b), "launch weight sums");
    }
    if (insert) {
        H2O_TRY(c, launch_insert_finish(a, n_kept), "launch insert-always score update");
        H2O_TRY(c, launch_scatter(a), "launch scatter");
    } else {
        H2O_TRY(c, launch_select(a), "launch select and copy");
    }
    c->last_T = T;
    c->last_n = n_kept;  // the step's cache candidates (all n, or the kept ones under insert-always)
    c->n = std::min<int64_t>(c->C, c->n + T);
    c->P += T;
    return H2O_OK;
}

int h2o_step(h2o_ctx* c, const void* q, const void* k, const void* v, void* out, int T, void* stream) {
    return step_impl(c, q, k, v, out, T, stream, false);
}

int h2o_prefill(h2o_ctx* c, const void* q, const void* k, const void* v, void* out, int T, int nchunks,
                void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (nchunks < 1 || T < 1) return fail(c, H2O_ERR_ARG, "need nchunks >= 1 and T >= 1 (got %d, %d)", nchunks, T);
    const size_t elem = c->dtype == H2O_FP32 ? 4 : 2;
    const size_t qb = (size_t)c->B * c->Hq * T * c->d * elem, kb = (size_t)c->B * c->Hkv * T * c->d * elem;
    for (int i = 0; i < nchunks; ++i) {
        rc = step_impl(c, q ? (const char*)q + i * qb : nullptr, k ? (const char*)k + i * kb : nullptr,
                       v ? (const char*)v + i * kb : nullptr, out ? (char*)out + i * qb : nullptr, T, stream, i > 0);
        if (rc != H2O_OK) return rc;
    }
    return H2O_OK;
}

int h2o_backward(h2o_ctx* c, const void* q, const void* k, const void* v, const float* lse, const void* dout,
                 int T, float* dq, float* dK, float* dV, float* dk, float* dv, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (T < 1) return fail(c, H2O_ERR_ARG, "T must be >= 1 (got %d)", T);
    if (!q || !k || !v || !lse || !dout || !dq || !dK || !dV || !dk || !dv)
        return fail(c, H2O_ERR_ARG, "every pointer argument must be non-NULL");
    for (const void* p : {q, k, v, dout, (const void*)lse, (const void*)dq, (const void*)dK, (const void*)dV,
                          (const void*)dk, (const void*)dv})
        if (!aligned16(p)) return fail(c, H2O_ERR_ALIGN, "every pointer argument must be 16-byte aligned");
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const int rows_pad = tc_rows_pad(c->Hq, c->Hkv, T);
    if (rows_pad > c->bwd_rows_pad) {
        // first use, or a longer chunk than before: (re)allocate once
        if (c->bwd_rows) {
            H2O_TRY(c, cudaStreamSynchronize(s), "sync before backward workspace growth");
            H2O_TRY(c, cudaDeviceSynchronize(), "sync before backward workspace growth");
            cudaFree(c->bwd_rows);
            c->bwd_rows = nullptr;
            c->bwd_rows_pad = 0;
        }
        H2O_TRY(c, cudaMalloc(&c->bwd_rows, sizeof(float) * 2 * (size_t)c->B * c->Hkv * rows_pad),
                "cudaMalloc(backward row tables)");
        c->bwd_rows_pad = rows_pad;
    }
    BwdArgs a{};
    a.B = c->B;
    a.Hq = c->Hq;
    a.Hkv = c->Hkv;
    a.d = c->d;
    a.C = c->C;
    a.T = T;
    a.n = (int)c->n;
    a.dtype = c->dtype;
    a.q = q;
    a.k = k;
    a.v = v;
    a.lse = lse;
    a.dout = dout;
    a.Kc = c->Kc;
    a.Vc = c->Vc;
    a.dq = dq;
    a.dKc = dK;
    a.dVc = dV;
    a.dk = dk;
    a.dv = dv;
    a.rows_pad = c->bwd_rows_pad;
    a.Drow = c->bwd_rows;
    a.L2row = c->bwd_rows + (size_t)c->B * c->Hkv * c->bwd_rows_pad;
    a.wb.err_word = c->err_dev;
    a.wb.ns = c->wait_ns;
    a.stream = s;
    a.num_sms = c->num_sms;
    LaunchLog local_log;
    a.log = &local_log;
    if (c->prof_on && c->prof_steps < c->prof_max_steps) {
        const int slot = c->prof_steps++;
        a.log = &c->prof_logs[slot];
        a.log->n = 0;
        a.log->ev = &c->prof_ev[(size_t)slot * (kMaxStepKernels + 1)];
        H2O_TRY(c, cudaEventRecord(a.log->ev[0], s), "record profiling event");
    }
    if (c->use_tc) {
        H2O_TRY(c, tc_backward(a), "launch tensor-core backward");
    } else {
        H2O_TRY(c, launch_bwd_simt(a), "launch backward");
    }
    return H2O_OK;
}

int h2o_step_host(h2o_ctx* c, const void* q, const void* k, const void* v, void* out, int T, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (T < 1) return fail(c, H2O_ERR_ARG, "T must be >= 1 (got %d)", T);
    if (!q || !k || !v || !out) return fail(c, H2O_ERR_ARG, "q, k, v, out must be non-NULL");
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t qb = (size_t)c->B * c->Hq * T * c->d * c->elem;
    const size_t kb = (size_t)c->B * c->Hkv * T * c->d * c->elem;
    auto up16 = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t need = up16(qb) * 2 + up16(kb) * 2;
    if (need > c->stage_bytes) {
        H2O_TRY(c, cudaStreamSynchronize(s), "sync before staging growth");
        cudaFree(c->stage);
        c->stage = nullptr;
        c->stage_bytes = 0;
        H2O_TRY(c, cudaMalloc(&c->stage, need), "cudaMalloc(staging)");
        c->stage_bytes = need;
    }
    char* base = (char*)c->stage;
    void* dq = base;
    void* dout = base + up16(qb);
    void* dk = base + 2 * up16(qb);
    void* dv = base + 2 * up16(qb) + up16(kb);
    H2O_TRY(c, cudaMemcpyAsync(dq, q, qb, cudaMemcpyHostToDevice, s), "copy q to device");
    H2O_TRY(c, cudaMemcpyAsync(dk, k, kb, cudaMemcpyHostToDevice, s), "copy k to device");
    H2O_TRY(c, cudaMemcpyAsync(dv, v, kb, cudaMemcpyHostToDevice, s), "copy v to device");
    rc = h2o_step(c, dq, dk, dv, dout, T, stream);
    if (rc != H2O_OK) return rc;
    H2O_TRY(c, cudaMemcpyAsync(out, dout, qb, cudaMemcpyDeviceToHost, s), "copy out to host");
    H2O_TRY(c, cudaStreamSynchronize(s), "synchronise after step");
    return check_ctx(c);
}


int h2o_step_host_async(h2o_ctx* c, const void* q, const void* k, const void* v, void* out, int T,
                        void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (T < 1) return fail(c, H2O_ERR_ARG, "T must be >= 1 (got %d)", T);
    if (!q || !k || !v || !out) return fail(c, H2O_ERR_ARG, "q, k, v, out must be non-NULL");
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t qb = (size_t)c->B * c->Hq * T * c->d * c->elem;
    const size_t kb = (size_t)c->B * c->Hkv * T * c->d * c->elem;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t need = up(qb) * 2 + up(kb) * 2;  // q, out, k, v
    if (!c->s_in) {
        H2O_TRY(c, cudaStreamCreateWithFlags(&c->s_in, cudaStreamNonBlocking), "create upload stream");
        H2O_TRY(c, cudaStreamCreateWithFlags(&c->s_out, cudaStreamNonBlocking), "create download stream");
        for (int i = 0; i < 2; ++i)
            for (cudaEvent_t* e : {&c->ev_in[i], &c->ev_step[i], &c->ev_out[i]})
                H2O_TRY(c, cudaEventCreateWithFlags(e, cudaEventDisableTiming), "create pipeline event");
    }
    if (need > c->aslot_bytes) {  // grow both slots once every queued copy is done
        H2O_TRY(c, cudaStreamSynchronize(c->s_in), "sync before staging growth");
        H2O_TRY(c, cudaStreamSynchronize(c->s_out), "sync before staging growth");
        H2O_TRY(c, cudaStreamSynchronize(s), "sync before staging growth");
        for (int i = 0; i < 2; ++i) {
            cudaFree(c->aslot[i]);
            c->aslot[i] = nullptr;
        }
        c->aslot_bytes = 0;
        for (int i = 0; i < 2; ++i) H2O_TRY(c, cudaMalloc(&c->aslot[i], need), "cudaMalloc(async staging)");
        c->aslot_bytes = need;
    }
    const int sl = (int)(c->achunks & 1);
    char* base = (char*)c->aslot[sl];
    void* dq = base;
    void* dout = base + up(qb);
    void* dk = base + 2 * up(qb);
    void* dv = base + 2 * up(qb) + up(kb);
    // upload, once the step two chunks back has finished reading this slot
    H2O_TRY(c, cudaStreamWaitEvent(c->s_in, c->ev_step[sl], 0), "order upload");
    H2O_TRY(c, cudaMemcpyAsync(dq, q, qb, cudaMemcpyHostToDevice, c->s_in), "copy q to device");
    H2O_TRY(c, cudaMemcpyAsync(dk, k, kb, cudaMemcpyHostToDevice, c->s_in), "copy k to device");
    H2O_TRY(c, cudaMemcpyAsync(dv, v, kb, cudaMemcpyHostToDevice, c->s_in), "copy v to device");
    H2O_TRY(c, cudaEventRecord(c->ev_in[sl], c->s_in), "record upload");
    // the step, once the inputs are there and the slot's last output is downloaded
    H2O_TRY(c, cudaStreamWaitEvent(s, c->ev_in[sl], 0), "order step");
    H2O_TRY(c, cudaStreamWaitEvent(s, c->ev_out[sl], 0), "order step");
    rc = h2o_step(c, dq, dk, dv, dout, T, stream);
    if (rc != H2O_OK) return rc;
    H2O_TRY(c, cudaEventRecord(c->ev_step[sl], s), "record step");
    // download
    H2O_TRY(c, cudaStreamWaitEvent(c->s_out, c->ev_step[sl], 0), "order download");
    H2O_TRY(c, cudaMemcpyAsync(out, dout, qb, cudaMemcpyDeviceToHost, c->s_out), "copy out to host");
    H2O_TRY(c, cudaEventRecord(c->ev_out[sl], c->s_out), "record download");
    ++c->achunks;
    return H2O_OK;
}

int h2o_set_policy(h2o_ctx* c, int policy) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    if (policy != H2O_POLICY_SUM && policy != H2O_POLICY_NORMALIZED && policy != H2O_POLICY_INSERT_ALWAYS)
        return fail(c, H2O_ERR_ARG, "unknown eviction policy %d", policy);
    if (policy == H2O_POLICY_INSERT_ALWAYS && !c->ins_K) {
        // all five buffers or none: a failed allocation leaves the context as
        // it was (policy unchanged, no buffer recorded), so a retry starts over
        DeviceGuard g(c->device);
        const size_t groups = (size_t)c->B * c->Hkv;
        const size_t rows = groups * c->C;
        void* bufs[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
        const size_t bytes[5] = {rows * c->d * c->elem, rows * c->d * c->elem, sizeof(int32_t) * rows,
                                 sizeof(float) * rows, sizeof(int32_t) * rows};
        for (int i = 0; i < 5; ++i) {
            const cudaError_t e = cudaMalloc(&bufs[i], bytes[i]);
            if (e != cudaSuccess) {
                for (int j = 0; j < i; ++j) cudaFree(bufs[j]);
                cudaGetLastError();  // an allocation failure is not sticky: clear it
                return fail(c, e == cudaErrorMemoryAllocation ? H2O_ERR_OOM : H2O_ERR_CUDA,
                            "cudaMalloc of the insert-always workspace (%zu bytes): %s", bytes[i],
                            cudaGetErrorString(e));
            }
        }
        c->ins_K = bufs[0];
        c->ins_V = bufs[1];
        c->ins_slot = static_cast<int32_t*>(bufs[2]);
        c->ins_score = static_cast<float*>(bufs[3]);
        c->ins_pos = static_cast<int32_t*>(bufs[4]);
    }
    c->policy = policy;
    return H2O_OK;
}

int h2o_host_sync(h2o_ctx* c) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    DeviceGuard g(c->device);
    if (c->s_in) {
        H2O_TRY(c, cudaStreamSynchronize(c->s_in), "synchronise uploads");
        H2O_TRY(c, cudaStreamSynchronize(c->s_out), "synchronise downloads");
    }
    return check_ctx(c);
}

int h2o_scores(h2o_ctx* c, float* dst, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (!dst) return fail(c, H2O_ERR_ARG, "dst is NULL");
    DeviceGuard g(c->device);
    H2O_TRY(c, cudaMemcpyAsync(dst, c->scores, sizeof(float) * c->B * c->Hkv * c->C, cudaMemcpyDeviceToDevice,
                               (cudaStream_t)stream), "copy scores");
    return H2O_OK;
}

int h2o_positions(h2o_ctx* c, int32_t* dst, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (!dst) return fail(c, H2O_ERR_ARG, "dst is NULL");
    DeviceGuard g(c->device);
    H2O_TRY(c, cudaMemcpyAsync(dst, c->pos, sizeof(int32_t) * c->B * c->Hkv * c->C, cudaMemcpyDeviceToDevice,
                               (cudaStream_t)stream), "copy positions");
    return H2O_OK;
}

int h2o_counters(const h2o_ctx* c, int64_t* P, int64_t* n) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    if (P) *P = c->P;
    if (n) *n = c->n;
    return H2O_OK;
}

int h2o_last_step_info(const h2o_ctx* c, int* T_last, int* n_prev) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    if (T_last) *T_last = c->last_T;
    if (n_prev) *n_prev = c->last_n;
    return H2O_OK;
}

int h2o_candidates(h2o_ctx* c, float* scores, int32_t* pos, uint8_t* kept, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (c->last_T == 0) return fail(c, H2O_ERR_ARG, "no step has run yet");
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t groups = (size_t)c->B * c->Hkv;
    const size_t nc = (size_t)c->last_n + c->last_T;
    const size_t src_pitch = (size_t)c->C + c->tmax;
    if (scores)
        H2O_TRY(c, cudaMemcpy2DAsync(scores, nc * 4, c->cand_score, src_pitch * 4, nc * 4, groups,
                                     cudaMemcpyDeviceToDevice, s), "copy candidate scores");
    if (pos)
        H2O_TRY(c, cudaMemcpy2DAsync(pos, nc * 4, c->cand_pos, src_pitch * 4, nc * 4, groups,
                                     cudaMemcpyDeviceToDevice, s), "copy candidate positions");
    if (kept)
        H2O_TRY(c, cudaMemcpy2DAsync(kept, nc, c->cand_kept, src_pitch, nc, groups, cudaMemcpyDeviceToDevice, s),
                "copy kept flags");
    return H2O_OK;
}

int h2o_token_slots(h2o_ctx* c, int32_t* dst, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (c->last_T == 0) return fail(c, H2O_ERR_ARG, "no step has run yet");
    if (!dst) return fail(c, H2O_ERR_ARG, "dst is NULL");
    DeviceGuard g(c->device);
    const size_t groups = (size_t)c->B * c->Hkv;
    H2O_TRY(c, cudaMemcpy2DAsync(dst, (size_t)c->last_T * 4, c->token_slot, (size_t)c->tmax * 4,
                                 (size_t)c->last_T * 4, groups, cudaMemcpyDeviceToDevice, (cudaStream_t)stream),
            "copy token slots");
    return H2O_OK;
}

int h2o_lse(h2o_ctx* c, float* dst, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (c->last_T == 0) return fail(c, H2O_ERR_ARG, "no step has run yet");
    if (!dst) return fail(c, H2O_ERR_ARG, "dst is NULL");
    DeviceGuard g(c->device);
    const size_t rows = (size_t)c->B * c->Hq;
    H2O_TRY(c, cudaMemcpy2DAsync(dst, (size_t)c->last_T * 4, c->lse, (size_t)c->tmax * 4, (size_t)c->last_T * 4,
                                 rows, cudaMemcpyDeviceToDevice, (cudaStream_t)stream), "copy lse");
    return H2O_OK;
}

int h2o_get_state(h2o_ctx* c, void* K, void* V, float* scores, int32_t* positions, int64_t* P, int64_t* n,
                  void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t groups = (size_t)c->B * c->Hkv;
    const size_t cb = groups * c->C * c->d * c->elem;
    if (K) H2O_TRY(c, cudaMemcpyAsync(K, c->Kc, cb, cudaMemcpyDeviceToDevice, s), "copy K");
    if (V) H2O_TRY(c, cudaMemcpyAsync(V, c->Vc, cb, cudaMemcpyDeviceToDevice, s), "copy V");
    if (scores) H2O_TRY(c, cudaMemcpyAsync(scores, c->scores, groups * c->C * 4, cudaMemcpyDeviceToDevice, s), "copy scores");
    if (positions) H2O_TRY(c, cudaMemcpyAsync(positions, c->pos, groups * c->C * 4, cudaMemcpyDeviceToDevice, s), "copy positions");
    if (P) *P = c->P;
    if (n) *n = c->n;
    return H2O_OK;
}

int h2o_set_state(h2o_ctx* c, const void* K, const void* V, const float* scores, const int32_t* positions,
                  int64_t P, int64_t n, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (!K || !V || !scores || !positions) return fail(c, H2O_ERR_ARG, "K, V, scores, positions must be non-NULL");
    if (P < 0 || P > (int64_t)INT32_MAX || n < 0 || n > c->C || n > P)
        return fail(c, H2O_ERR_ARG, "need 0 <= n <= min(C, P) and P < 2^31");
    DeviceGuard g(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t groups = (size_t)c->B * c->Hkv;
    std::vector<int32_t> hp(groups * c->C);
    H2O_TRY(c, cudaMemcpyAsync(hp.data(), positions, hp.size() * 4, cudaMemcpyDeviceToHost, s), "read positions");
    H2O_TRY(c, cudaStreamSynchronize(s), "sync set_state");
    std::vector<int32_t> sorted((size_t)n);
    for (size_t gi = 0; gi < groups; ++gi) {
        const int32_t* p = hp.data() + gi * c->C;
        for (int64_t j = 0; j < n; ++j) {
            if (p[j] < 0 || p[j] >= P)
                return fail(c, H2O_ERR_ARG, "group %zu slot %lld: position %d outside [0, P)", gi, (long long)j, p[j]);
            sorted[j] = p[j];
        }
        for (int64_t j = n; j < c->C; ++j)
            if (p[j] != -1) return fail(c, H2O_ERR_ARG, "group %zu slot %lld beyond n must be empty (-1)", gi, (long long)j);
        std::sort(sorted.begin(), sorted.end());
        if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end())
            return fail(c, H2O_ERR_ARG, "group %zu has duplicate positions", gi);
    }
    const size_t cb = groups * c->C * c->d * c->elem;
    H2O_TRY(c, cudaMemcpyAsync(c->Kc, K, cb, cudaMemcpyDeviceToDevice, s), "copy K");
    H2O_TRY(c, cudaMemcpyAsync(c->Vc, V, cb, cudaMemcpyDeviceToDevice, s), "copy V");
    H2O_TRY(c, cudaMemcpyAsync(c->scores, scores, groups * c->C * 4, cudaMemcpyDeviceToDevice, s), "copy scores");
    H2O_TRY(c, cudaMemcpyAsync(c->pos, positions, groups * c->C * 4, cudaMemcpyDeviceToDevice, s), "copy positions");
    c->P = P;
    c->n = n;
    c->last_T = 0;
    return H2O_OK;
}

int h2o_sync_check(h2o_ctx* c, void* stream) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    DeviceGuard g(c->device);
    H2O_TRY(c, cudaStreamSynchronize((cudaStream_t)stream), "synchronise");
    return check_ctx(c);
}

int h2o_profile_begin(h2o_ctx* c, int max_steps) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    if (max_steps < 1) return fail(c, H2O_ERR_ARG, "max_steps must be >= 1");
    DeviceGuard g(c->device);
    for (cudaEvent_t e : c->prof_ev) cudaEventDestroy(e);
    c->prof_ev.assign((size_t)max_steps * (kMaxStepKernels + 1), nullptr);
    for (auto& e : c->prof_ev) H2O_TRY(c, cudaEventCreate(&e), "cudaEventCreate");
    c->prof_logs.assign(max_steps, LaunchLog());
    c->prof_max_steps = max_steps;
    c->prof_steps = 0;
    c->prof_on = true;
    return H2O_OK;
}

int h2o_profile_end(h2o_ctx* c, int max_kernels, const char** names, double* total_ms, int* launches) {
    if (!c) return fail(nullptr, H2O_ERR_ARG, "null context");
    if (!c->prof_on) return fail(c, H2O_ERR_ARG, "profiling was not started");
    DeviceGuard g(c->device);
    c->prof_on = false;
    int nk = 0;
    std::vector<const char*> nm;
    std::vector<double> ms;
    std::vector<int> cnt;
    for (int st = 0; st < c->prof_steps; ++st) {
        const LaunchLog& L = c->prof_logs[st];
        for (int i = 0; i < L.n; ++i) {
            cudaEvent_t a = c->prof_ev[(size_t)st * (kMaxStepKernels + 1) + i];
            cudaEvent_t b = c->prof_ev[(size_t)st * (kMaxStepKernels + 1) + i + 1];
            H2O_TRY(c, cudaEventSynchronize(b), "cudaEventSynchronize");
            float t = 0.f;
            H2O_TRY(c, cudaEventElapsedTime(&t, a, b), "cudaEventElapsedTime");
            int idx = -1;
            for (int j = 0; j < (int)nm.size(); ++j)
                if (strcmp(nm[j], L.names[i]) == 0) idx = j;
            if (idx < 0) {
                nm.push_back(L.names[i]);
                ms.push_back(0.0);
                cnt.push_back(0);
                idx = (int)nm.size() - 1;
            }
            ms[idx] += t;
            cnt[idx] += 1;
        }
    }
    for (cudaEvent_t e : c->prof_ev) cudaEventDestroy(e);
    c->prof_ev.clear();
    c->prof_logs.clear();
    nk = (int)nm.size();
    for (int j = 0; j < nk && j < max_kernels; ++j) {
        if (names) names[j] = nm[j];
        if (total_ms) total_ms[j] = ms[j];
        if (launches) launches[j] = cnt[j];
    }
    return nk;
}

int h2o_selftest_exp2(const float* x, float* y_poly3, float* y_poly4, float* y_mufu, int n, void* stream) {
    if (n < 0 || (n > 0 && (!x || !y_poly3 || !y_poly4 || !y_mufu)))
        return fail(nullptr, H2O_ERR_ARG, "h2o_selftest_exp2: bad arguments");
    if (n == 0) return H2O_OK;
    H2O_TRY(nullptr, tc_exp2_selftest(x, y_poly3, y_poly4, y_mufu, n, (cudaStream_t)stream),
            "launch exp2 self-test");
    return H2O_OK;
}

int h2o_selftest_wait(h2o_ctx* c, int spins, void* stream) {
    int rc = check_ctx(c);
    if (rc != H2O_OK) return rc;
    DeviceGuard g(c->device);
    WaitBound wb;
    wb.err_word = c->err_dev;
    wb.ns = (unsigned long long)(spins > 0 ? spins : 1) * 1000000ull;  // spins read as milliseconds
    H2O_TRY(c, launch_wait_selftest(wb, (cudaStream_t)stream), "launch wait self-test");
    H2O_TRY(c, cudaStreamSynchronize((cudaStream_t)stream), "synchronise wait self-test");
    return check_ctx(c);
}

}  // extern "C"
