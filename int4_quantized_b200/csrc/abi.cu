// abi.cu -- the extern "C" entry points declared in include/q4.h.
//
// Every call validates its arguments on the host before enqueuing anything, then
// launches the kernels on the caller's stream. Nothing is allocated here; the only state
// that survives a call is qgemm_noalloc's cached scratch address per device.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "kernels.h"

namespace q4 {

// The last failing CUDA call of this host thread, for q4_last_cuda_error().
thread_local char g_last_cuda_error[160] = "";

q4_status cuda_error(cudaError_t e, const char *where) {
    if (e == cudaSuccess) return Q4_OK;
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s (%s)", where, cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return Q4_ERR_CUDA;
}

// rowscale.cu: out[n] = scales[n / rows_per_scale] for n < N
cudaError_t launch_expand_row_scales(const float *scales, int64_t rows_per_scale, int64_t N, float *out,
                                     cudaStream_t st);
}  // namespace q4

namespace {

// qgemm's task split is planned for a full B200 (148 SMs) whatever device runs it, so
// the workspace size is a pure function of the problem and needs no CUDA call.
constexpr int kPlanSMs = 148;

inline int device_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool mul_ok(int64_t a, int64_t b, int64_t *out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

q4_status check_format(int64_t rows, int64_t cols, int bits, int64_t group, int64_t *n) {
    if (bits != 4 && bits != 8) return Q4_ERR_ARG;
    if (group < 1) return Q4_ERR_ARG;
    if (!mul_ok(rows, cols, n)) return Q4_ERR_ARG;
    if (*n % group != 0) return Q4_ERR_ARG;
    if (bits == 4 && (*n % 2) != 0) return Q4_ERR_ARG;
    return Q4_OK;
}

inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }

inline q4_status cuda_status(cudaError_t e, const char *where) { return q4::cuda_error(e, where); }

// Path selection and workspace layout of one qgemm call.
struct QgemmPlan {
    q4::GemvPlan gemv;    // the fused GEMV plan (for the row-scale group when rps > 1)
    int64_t group;        // group the kernels see: the caller's, or K for groups of whole rows
    int64_t rps;          // rows per scale when the group spans whole rows, else 1
    bool prefill;         // bf16 x, M >= 64: the tensor-core GEMM
    bool any;             // a group neither fast path takes: the any-group kernel (no workspace)
    size_t scale_bytes;   // expanded per-row scales at the start of the workspace (rps > 1)
    size_t total_bytes;   // workspace the call needs
};

// Returns Q4_OK and fills the plan, or the reason the call cannot run. Groups that divide
// K (in multiples of 32) run on the fused GEMV or the tensor-core GEMM; groups of whole
// rows too, once their scales are expanded to one per row in the workspace; every other
// divisor of N * K (and any K) runs on the any-group kernel.
q4_status plan_qgemm(int64_t M, int64_t N, int64_t K, int bits, int64_t group, q4_xdtype xt, QgemmPlan *p) {
    if (bits != 4 && bits != 8) return Q4_ERR_ARG;
    if (M < 0 || N < 0 || K < 1 || group < 1) return Q4_ERR_ARG;
    if (xt != Q4_X_F32 && xt != Q4_X_BF16) return Q4_ERR_ARG;
    if (N > 0 && (N > ((int64_t)1 << 40) / K || (N * K) % group != 0)) return Q4_ERR_ARG;  // no such packed tensor
    if (bits == 4 && (N * K) % 2 != 0) return Q4_ERR_ARG;                               // (qpack's rule)
    p->group = group;
    p->rps = 1;
    p->any = false;
    p->prefill = false;
    if (K % group != 0) {
        if (group % K == 0) {
            p->rps = group / K;
            p->group = K;
        } else {
            p->any = true;
        }
    }
    // the fused paths take K and groups in multiples of 32 (groups of whole rows as K)
    if (!p->any && (K % 32 != 0 || p->group % 32 != 0)) {
        p->any = true;
        p->group = group;
        p->rps = 1;
    }
    if (!p->any && !q4::gemv_plan(M > 0 ? M : 1, N > 0 ? N : 1, K, bits, p->group, xt == Q4_X_BF16, kPlanSMs,
                                  &p->gemv))
        return Q4_ERR_UNSUPPORTED;
    if (p->any) {
        p->scale_bytes = p->total_bytes = 0;
        return Q4_OK;
    }
    p->prefill = q4::prefill_supported(M, N, K, bits, p->group, xt == Q4_X_BF16);
    p->scale_bytes = p->rps > 1 ? align256((size_t)N * 4) : 0;
    p->total_bytes = p->scale_bytes + (p->prefill ? 0 : p->gemv.bytes);
    return Q4_OK;
}

// Scratch of qgemm_noalloc: one file-scope device array per device, created with the
// module; its address is looked up once per device and cached.
constexpr size_t kNoAllocBytes = Q4_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

q4_status noalloc_scratch(void **out) {
    int dev = -1;
    const cudaError_t ge = cudaGetDevice(&dev);
    if (ge != cudaSuccess) return cuda_status(ge, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return Q4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return Q4_OK;
}

}  // namespace

extern "C" {

int q4_version(void) { return 200; }

const char *q4_last_cuda_error(void) { return q4::g_last_cuda_error; }

const char *q4_status_str(q4_status s) {
    switch (s) {
        case Q4_OK: return "ok";
        case Q4_ERR_ARG: return "invalid argument";
        case Q4_ERR_UNSUPPORTED: return "shape or format not covered by this kernel";
        case Q4_ERR_CUDA: return "CUDA error";
        case Q4_ERR_NONFINITE: return "non-finite weight in a group";
        case Q4_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case Q4_ERR_SCRATCH_LIMIT: return "problem needs more scratch than qgemm_noalloc's built-in buffer";
    }
    return "unknown status";
}

size_t q4_payload_bytes(int64_t rows, int64_t cols, int bits) {
    int64_t n;
    if ((bits != 4 && bits != 8) || !mul_ok(rows, cols, &n)) return 0;
    if (bits == 4 && n % 2) return 0;
    return (size_t)(bits == 8 ? n : n / 2);
}

int64_t q4_num_scales(int64_t rows, int64_t cols, int64_t group) {
    int64_t n;
    if (group < 1 || !mul_ok(rows, cols, &n) || n % group) return -1;
    return n / group;
}

q4_status qpack(const float *w, int64_t rows, int64_t cols, int bits, int64_t group,
                uint8_t *payload, float *scales, uint32_t *status_word, void *stream) {
    int64_t n;
    q4_status st = check_format(rows, cols, bits, group, &n);
    if (st != Q4_OK) return st;
    if (n == 0) return Q4_OK;
    if (!w || !payload || !scales) return Q4_ERR_ARG;
    cudaError_t e = q4::launch_qpack(w, n, bits, group, payload, scales, status_word,
                                     as_stream(stream), device_sms());
    return cuda_status(e, "qpack launch");
}

q4_status qdequant(const uint8_t *payload, const float *scales, int64_t rows, int64_t cols,
                   int bits, int64_t group, float *w_out, void *stream) {
    int64_t n;
    q4_status st = check_format(rows, cols, bits, group, &n);
    if (st != Q4_OK) return st;
    if (n == 0) return Q4_OK;
    if (!payload || !scales || !w_out) return Q4_ERR_ARG;
    cudaError_t e = q4::launch_qdequant(payload, scales, n, bits, group, w_out, as_stream(stream),
                                        device_sms());
    return cuda_status(e, "qdequant launch");
}

size_t q4_qgemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int64_t group,
                                q4_xdtype xt) {
    QgemmPlan p;
    if (plan_qgemm(M, N, K, bits, group, xt, &p) != Q4_OK) return 0;
    return p.total_bytes;
}

q4_status qgemm_ex(const void *x, q4_xdtype xt, int64_t M, const uint8_t *payload,
                   const float *scales, int64_t N, int64_t K, int bits, int64_t group, float *y,
                   void *workspace, size_t workspace_bytes, uint32_t flags, uint32_t *status_word,
                   void *stream) {
    if (flags & ~(uint32_t)Q4_QGEMM_WEIGHTS_STATIC) return Q4_ERR_ARG;
    QgemmPlan p;
    q4_status st = plan_qgemm(M, N, K, bits, group, xt, &p);
    if (st != Q4_OK) return st;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !payload || !scales || !y) return Q4_ERR_ARG;
    if (p.any) {
        const cudaError_t ae = q4::launch_any_group(x, xt == Q4_X_BF16, M, payload, scales, N, K, bits, group, y,
                                                    device_sms(), as_stream(stream));
        return cuda_status(ae, "any-group launch");
    }
    if ((uintptr_t)payload % 16 || (uintptr_t)x % 16) return Q4_ERR_UNSUPPORTED;
    if ((!p.prefill || p.total_bytes > 0) && (uintptr_t)workspace % 256) return Q4_ERR_WORKSPACE;
    if (p.total_bytes > 0 && (!workspace || workspace_bytes < p.total_bytes)) return Q4_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    const float *sc = scales;
    bool early = (flags & Q4_QGEMM_WEIGHTS_STATIC) != 0;
    if (p.rps > 1) {
        // one scale per row, written by the kernel just before: no early start
        float *rs = static_cast<float *>(workspace);
        const cudaError_t re = q4::launch_expand_row_scales(scales, p.rps, N, rs, s);
        if (re != cudaSuccess) return cuda_status(re, "row-scale launch");
        sc = rs;
        early = false;
    }
    cudaError_t e;
    if (p.prefill) {
        e = q4::launch_prefill(x, M, payload, sc, N, K, bits, p.group, y, status_word, device_sms(), s);
    } else {
        void *ws = p.gemv.bytes ? static_cast<char *>(workspace) + p.scale_bytes : nullptr;
        e = q4::launch_gemv(p.gemv, x, xt == Q4_X_BF16, M, payload, sc, N, K, p.group, y, ws, status_word, early,
                            s);
    }
    return cuda_status(e, p.prefill ? "prefill launch" : "gemv launch");
}

q4_status qgemm(const void *x, q4_xdtype xt, int64_t M, const uint8_t *payload,
                const float *scales, int64_t N, int64_t K, int bits, int64_t group, float *y,
                void *workspace, size_t workspace_bytes, uint32_t *status_word, void *stream) {
    return qgemm_ex(x, xt, M, payload, scales, N, K, bits, group, y, workspace, workspace_bytes, 0u,
                    status_word, stream);
}

q4_status qgemm_noalloc(const void *x, q4_xdtype xt, int64_t M, const uint8_t *payload,
                        const float *scales, int64_t N, int64_t K, int bits, int64_t group,
                        float *y, uint32_t *status_word, void *stream) {
    QgemmPlan p;
    q4_status st = plan_qgemm(M, N, K, bits, group, xt, &p);
    if (st != Q4_OK) return st;
    if (M == 0 || N == 0) return Q4_OK;
    if (p.total_bytes > kNoAllocBytes) return Q4_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != Q4_OK) return st;
    return qgemm(x, xt, M, payload, scales, N, K, bits, group, y, scratch, kNoAllocBytes,
                 status_word, stream);
}

}  // extern "C"
