// kernels.h -- internal launch interface between the C ABI (abi.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/q4.h"

namespace q4 {

// Records e (with the failing step) for q4_last_cuda_error(); Q4_OK when e is cudaSuccess,
// else Q4_ERR_CUDA.
q4_status cuda_error(cudaError_t e, const char *where);

cudaError_t launch_qpack(const float *w, int64_t n, int bits, int64_t group, uint8_t *payload,
                         float *scales, uint32_t *status, cudaStream_t st, int sms);
cudaError_t launch_qdequant(const uint8_t *payload, const float *scales, int64_t n, int bits,
                            int64_t group, float *out, cudaStream_t st, int sms);

// ---- decode GEMV --------------------------------------------------------------------
// Plan of one GEMV call: how K is cut into segments (one 128/64/32-bit load per lane per
// weight row), how a thread-block cluster splits K, and where the activation pieces live.
struct GemvPlan {
    int bits, L;        // L = bytes each lane reads per weight row per segment (16, 8 or 4)
    int P;              // bf16 pieces per activation: 3 for fp32 x, 1 for bf16 x
    int segk;           // k per segment = 32 * L / bits
    int segs;           // segments per row = K / segk
    int spg;            // segments per scale group = group / segk
    int gps;            // groups per stage (divides it), 0 (stage inside a group) or -1
    int NB;             // n8 blocks of MMA columns per 16-row chunk of x (1, 2, 3, 4 or 6)
    int lw;             // piece lanes stored per (MMA, n8 block): 16 or 32
    int paired;         // pieces of two consecutive MMAs interleaved
    int clusters;       // CTAs along N = ceil(N / 128)
    int CS;             // CTAs per cluster = splits of K (1..8)
    int ctas_per_sm;    // 2, or 1 when the piece slots are large
    int stages_total;   // 128-byte tiles per weight row
    int stages_per_cta; // tiles per CTA's K range
    int ebs, n_eb;      // tiles per k-block (scale staging block), k-blocks per row
    int nst_ring;       // ring depth
    int fslot_bytes;    // piece bytes of one stage
    int ink;            // one row of x: pieces built in shared memory, no workspace
    int hyb;            // one row of x, regular groups: per stage, exact digits or pieces
    int nmc;            // 16-row chunks of x = ceil(M / 16)
    size_t smem_bytes;  // dynamic shared memory per CTA
    size_t off_frag, bytes;  // workspace layout and size (0 when ink)
};

// Returns false when this GEMV does not cover (bits, group, K).
bool gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int64_t group, bool x_bf16, int sms, GemvPlan *pl);

cudaError_t launch_gemv(const GemvPlan &pl, const void *x, bool x_bf16, int64_t M,
                        const uint8_t *payload, const float *scales, int64_t N, int64_t K,
                        int64_t group, float *y, void *ws, uint32_t *status, bool weights_static,
                        cudaStream_t st);

// ---- tensor maps ------------------------------------------------------------------------
// cuTensorMapEncodeTiled, fetched from the driver at run time (nullptr if unavailable).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();
// The GEMV's map of an [N][K*bits/8] payload: tiles of box_rows rows x 128 bytes, 128B swizzle.
bool encode_payload_map(CUtensorMap *tm, const uint8_t *payload, int64_t N, int64_t K, int bits, int box_rows);

// ---- prefill GEMM (tcgen05) ----------------------------------------------------------
// bf16 x with M >= 64, K and group multiples of 64: the tensor-memory GEMM of prefill.cu.
bool prefill_supported(int64_t M, int64_t N, int64_t K, int bits, int64_t group, bool x_bf16);
cudaError_t launch_prefill(const void *x, int64_t M, const uint8_t *payload, const float *scales, int64_t N,
                           int64_t K, int bits, int64_t group, float *y, uint32_t *status, int sms,
                           cudaStream_t st);

// ---- any group (anygroup.cu) ------------------------------------------------------------
// Groups the two paths above do not take: any divisor of N * K (crossing rows at varying
// offsets, or narrower than 32), any K; exact fp32 w', fp64 sums.
cudaError_t launch_any_group(const void *x, bool x_bf16, int64_t M, const uint8_t *payload, const float *scales,
                             int64_t N, int64_t K, int bits, int64_t group, float *y, int sms, cudaStream_t st);

}  // namespace q4
