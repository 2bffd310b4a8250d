// mru_noalloc.cu -- mru_scan_fused_noalloc: the fused scan without a
// caller-supplied workspace, for callers that may not allocate device memory
// at all (for example a plugin running inside a host framework that owns
// every device allocation, or a service that reserves its whole memory budget
// at start-up and forbids allocation afterwards).  Its scratch lives in one
// fixed-size, file-scope __device__ array instead.
#include <string.h>

#include "mru_internal.cuh"

namespace {

// The scratch every call of mru_scan_fused_noalloc uses.  Every GPU whose
// context loads this library holds these bytes until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[MRU_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code
// the symbol is only a host-side stand-in, so the address is asked for with
// cudaGetSymbolAddress, with the device current, on every call (a cheap
// lookup); nothing is cached, so a context torn down and created again
// (cudaDeviceReset) gets the address of its own copy of the array.
cudaError_t scratch_address(void** out)
{
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" mru_status mru_scan_fused_noalloc(const mru_problem* p, const void* x, const float* S0,
                                             const mru_readout* ro, float* S_out, float* o_out,
                                             uint32_t* status_out, void* stream)
{
    using namespace mru;
    if (!p) return MRU_ERR_INVALID_ARG;
    mru_problem q = *p;
    if (fused_workspace_bytes(q, ro) == 0) {
        // invalid problem: let the shared validation name the error
        return mru_scan_fused(&q, x, S0, ro, S_out, o_out, nullptr, 0, stream);
    }
    // Pick the chunk: the caller's, else the library's choice doubled until
    // the workspace of this very call (its source, output form and readout
    // layout) fits the fixed scratch.
    if (q.chunk == 0) {
        q.chunk = mru_chosen_chunk(&q, ro != nullptr);
        while (fused_workspace_bytes(q, ro) > MRU_NOALLOC_SCRATCH_BYTES && (int64_t)q.chunk < q.L &&
               q.chunk < (1 << 30))
            q.chunk *= 2;
    }
    if (fused_workspace_bytes(q, ro) > MRU_NOALLOC_SCRATCH_BYTES) return MRU_ERR_WORKSPACE;
    if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u)) return MRU_ERR_INVALID_ARG;

    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return MRU_ERR_CUDA;
    // mru_scan_fused clears the status word itself and writes every other
    // scratch byte before reading it, so nothing left by an earlier call leaks in.
    mru_status st = mru_scan_fused(&q, x, S0, ro, S_out, o_out, ws, MRU_NOALLOC_SCRATCH_BYTES, stream);
    if (st != MRU_OK) return st;
    if (status_out) {
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        if (cudaMemcpyAsync(status_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return MRU_ERR_CUDA;
    }
    return MRU_OK;
}
