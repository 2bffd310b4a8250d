// mru_readout_bwd.cu -- the backward of the readout form: the upstream
// gradient of every state when the outputs are o_t = S_t U (and snapshots
// S_t every `every` steps), dL/dS_t = do_t U^T (+ the snapshot's gradient).
#include "mru_internal.cuh"

namespace mru {
namespace {

// dS[b, t, h] = do_t U_h^T (+ dP_k at 1-based t = k * every): one CTA per
// token-head row at a time (grid-stride over the B L H rows), do_t ([n, q])
// and the head's U_h ([n, q], u + h * u_hs) staged in shared memory, the
// row's n * n outputs written by consecutive threads.
__global__ void __launch_bounds__(256)
k_readout_grad(int64_t B, int64_t L, int64_t H, int n, int q, int64_t u_hs, const float* __restrict__ u,
               const float* __restrict__ d_o, int64_t every, const float* __restrict__ d_snap, float* __restrict__ dS)
{
    extern __shared__ float rsm[];
    float* sO = rsm;                                         // do_t, [n][q]
    float* sU = rsm + n * q;                                 // U_h, [n][q]
    const int nn = n * n, nq = n * q, ln = __ffs(n) - 1;  // n is a power of two
    const int64_t rows = B * L * H, L_s = every > 0 ? L / every : 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {   // row = (b L + t) H + h
        const int64_t h = row % H, bt = row / H, t = bt % L, b = bt / L;
        __syncthreads();                                     // the previous row's reads are done
        for (int e = threadIdx.x; e < nq; e += blockDim.x) {
            sO[e] = d_o[row * nq + e];
            sU[e] = u[h * u_hs + e];
        }
        __syncthreads();
        const float* snap = (d_snap && every > 0 && (t + 1) % every == 0)
                                ? d_snap + ((b * L_s + (t + 1) / every - 1) * H + h) * nn
                                : nullptr;
        float* out = dS + row * nn;
        for (int e = threadIdx.x; e < nn; e += blockDim.x) {
            const int i = e >> ln, j = e & (n - 1);
            float a = 0.0f;
            for (int c = 0; c < q; ++c) a = fmaf(sO[i * q + c], sU[j * q + c], a);
            if (snap) a += snap[e];
            out[e] = a;
        }
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
    const int64_t rows = p.B * p.L * p.H;
    const int64_t blocks = rows < (int64_t)sms * 8 ? rows : (int64_t)sms * 8;
    const size_t sm = sizeof(float) * 2 * (size_t)p.n * q;
    k_readout_grad<<<(unsigned)blocks, 256, sm, s>>>(p.B, p.L, p.H, p.n, q, u_hs, u, d_o, every, d_snap, dS);
    return cudaGetLastError();
}

}  // namespace mru
