// mru_internal.cuh -- shared device-side definitions of libmru (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mru.h"

namespace mru {

// Source of the per-token matrices a kernel consumes.
enum Source : int32_t {
    SRC_EMBEDDING = 0,   // construct X from the embedding x (mode, alpha, ...)
    SRC_X = 1,           // read X, use F = X - I
    SRC_F = 2            // read F = X - I directly
};

// Bits of the device status word (first 4 bytes of the workspace).
enum : uint32_t { STATUS_SINGULAR = 1u, STATUS_TIMEOUT = 2u };

// Everything a kernel needs to know about the problem, by value.
struct KParams {
    int64_t B, H, L;
    int32_t n;
    int32_t x_dtype;
    int32_t mode;
    int32_t src;
    float alpha;
    int32_t add_identity;
    float ldu_a;
    float ldu_d;
    int32_t math;        // mru_math requested
    int32_t chunk;       // tokens per chunk (C)
    int64_t K;           // chunks per sequence, ceil(L / C)
    int32_t group;       // chunk totals per carry group (G)
    int64_t NG;          // carry groups per sequence, ceil(K / G)
};

// Workspace carve-up (byte offsets from the workspace base).
struct Workspace {
    size_t status;       // uint32 status word
    size_t totals;       // float  [B*H, K, n, n]   chunk totals, split form (T - I)
    size_t local;        // double [B*H, K, n, n]   inclusive in-group prefixes of totals, split form
    size_t gcarry;       // double [B*H, NG, n, n]  exclusive group carries (full matrices)
    size_t carry;        // float  [B*H, K, n, n]   exclusive chunk carries (full matrices)
    size_t bytes;        // total
};

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Benchmark hook (mru_api.cu): records the caller's event for kernel slot
// `kernel`, before (after = 0) or after (after = 1) its launch; no-op when
// no events are registered.
void profile_mark(int kernel, int after, cudaStream_t s);

// n = 16 tensor-core kernels (mru_n16.cu).
namespace n16 {
int chunk_tokens();
bool supports(const KParams& p, bool readout);
cudaError_t launch_chunk(const KParams& p, const float* x, float* S_out, float* totals, uint32_t* status,
                         cudaStream_t s);
cudaError_t launch_fixup(const KParams& p, const float* carry, float* S_out, cudaStream_t s);
}  // namespace n16

// Launchers (mru_scan_v1.cu).
cudaError_t launch_build_states(const KParams& p, const void* x, float* X_out, int store_minus_identity,
                                void* ws_base, const Workspace& W, cudaStream_t s);
cudaError_t launch_scan(const KParams& p, const void* src, const float* S0, const float* u,
                        int64_t snap_every, float* S_out, float* o_out, float* snaps,
                        void* ws_base, const Workspace& W, cudaStream_t s, int* launches);
// Name of the i-th kernel one launch_scan call starts for this problem.
const char* kernel_name(const KParams& p, bool readout, int i);

}  // namespace mru
