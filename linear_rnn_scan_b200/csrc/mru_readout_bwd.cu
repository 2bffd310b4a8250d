// mru_readout_bwd.cu -- the backward of the readout form: the upstream
// gradient of every state when the outputs are o_t = S_t U (and snapshots
// S_t every `every` steps), dL/dS_t = do_t U^T (+ the snapshot's gradient).
#include "mru_internal.cuh"

namespace mru {
namespace {

// dS[b, t, h] = do_t U_h^T (+ dP_k at 1-based t = k * every): one thread per
// output element, grid-stride.  do_t is [n, q] per token and head, U_h the
// head's [n, q] query columns (u + h * u_hs).
__global__ void __launch_bounds__(256)
k_readout_grad(int64_t B, int64_t L, int64_t H, int n, int q, int64_t u_hs, const float* __restrict__ u,
               const float* __restrict__ d_o, int64_t every, const float* __restrict__ d_snap, float* __restrict__ dS)
{
    const int64_t nn = (int64_t)n * n, total = B * L * H * nn;
    const int64_t L_s = every > 0 ? L / every : 0;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = idx % nn, row = idx / nn;          // row = (b L + t) H + h
        const int i = (int)(e / n), j = (int)(e % n);
        const int64_t h = row % H, bt = row / H, t = bt % L, b = bt / L;
        const float* dO = d_o + row * n * q + (int64_t)i * q;
        const float* U = u + h * u_hs + (int64_t)j * q;
        float a = 0.0f;
        for (int c = 0; c < q; ++c) a = fmaf(dO[c], U[c], a);
        if (d_snap && every > 0 && (t + 1) % every == 0)
            a += d_snap[((b * L_s + (t + 1) / every - 1) * H + h) * nn + e];
        dS[idx] = a;
    }
}

}  // namespace

cudaError_t launch_readout_grad(const KParams& p, const float* u, int q, int64_t u_hs, const float* d_o,
                                int64_t every, const float* d_snap, float* dS, cudaStream_t s)
{
    const int64_t total = p.B * p.L * p.H * (int64_t)p.n * p.n;
    if (total == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    k_readout_grad<<<(unsigned)blocks, 256, 0, s>>>(p.B, p.L, p.H, p.n, q, u_hs, u, d_o, every, d_snap, dS);
    return cudaGetLastError();
}

}  // namespace mru
