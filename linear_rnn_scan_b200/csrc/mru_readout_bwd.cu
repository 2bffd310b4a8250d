// mru_readout_bwd.cu -- the backward of the readout form: the upstream
// gradient of every state when the outputs are o_t = S_t U (and snapshots
// S_t every `every` steps), dL/dS_t = do_t U^T (+ the snapshot's gradient).
#include "mru_internal.cuh"

namespace mru {
namespace {

// dS[b, t, h] = do_t U_h^T (+ dP_k at 1-based t = k * every): each thread
// writes float4 runs of one token-head row; a block takes one row at a time
// for n >= 32 and 256 / (n^2 / 4) rows at once below.  do_t ([n, q]) comes
// through the read-only cache (at most two rows i per warp: broadcasts).
// StageU: the heads' U_h ([n, q] = u + h * u_hs; one U when u_hs = 0) are
// staged transposed in shared memory once per block, [head][c][j], so each
// column c is a float4 read; otherwise U is read through the read-only cache
// (the heads' U too large to stage).
template <bool StageU>
__global__ void __launch_bounds__(256)
k_readout_grad(int64_t B, int64_t L, int64_t H, int n, int q, int64_t u_hs, const float* __restrict__ u,
               const float* __restrict__ d_o, int64_t every, const float* __restrict__ d_snap, float* __restrict__ dS)
{
    extern __shared__ __align__(16) float sUt[];
    const int nn = n * n, nq = n * q, ln = __ffs(n) - 1;   // n is a power of two, at least 4
    if constexpr (StageU) {
        const int heads = u_hs == 0 ? 1 : (int)H;
        for (int e = threadIdx.x; e < heads * nq; e += blockDim.x) {
            const int hh = e / nq, r = e - hh * nq, c = r >> ln, j = r & (n - 1);
            sUt[e] = u[hh * u_hs + j * q + c];
        }
        __syncthreads();
    }
    const int per_row = nn >> 2;                             // float4 runs of a row
    const int rpi = per_row >= 256 ? 1 : 256 / per_row;      // rows a block takes at a time
    const int lr = per_row >= 256 ? 0 : (int)threadIdx.x / per_row;
    const int e4_0 = per_row >= 256 ? (int)threadIdx.x : (int)threadIdx.x % per_row;
    const int e4_step = per_row >= 256 ? 256 : per_row;
    const int64_t rows = B * L * H, L_s = every > 0 ? L / every : 0;
    for (int64_t r0 = (int64_t)blockIdx.x * rpi; r0 < rows; r0 += (int64_t)gridDim.x * rpi) {
        const int64_t row = r0 + lr;                          // row = (b L + t) H + h
        if (row >= rows) continue;
        const int64_t h = row % H, bt = row / H, t = bt % L, b = bt / L;
        const float* dO = d_o + row * nq;
        const float* U = u + h * u_hs;
        const float* Ut = sUt + (u_hs == 0 ? 0 : (int)h * nq);
        const float4* snap = (d_snap && every > 0 && (t + 1) % every == 0)
                                 ? reinterpret_cast<const float4*>(d_snap + ((b * L_s + (t + 1) / every - 1) * H + h) * nn)
                                 : nullptr;
        float4* out = reinterpret_cast<float4*>(dS + row * nn);
        for (int e4 = e4_0; e4 < per_row; e4 += e4_step) {
            const int e = e4 << 2, i = e >> ln, j = e & (n - 1);
            float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
            for (int c = 0; c < q; ++c) {
                const float d = __ldg(dO + i * q + c);
                if constexpr (StageU) {
                    const float4 uv = *reinterpret_cast<const float4*>(Ut + c * n + j);
                    a0 = fmaf(d, uv.x, a0);
                    a1 = fmaf(d, uv.y, a1);
                    a2 = fmaf(d, uv.z, a2);
                    a3 = fmaf(d, uv.w, a3);
                } else {
                    a0 = fmaf(d, __ldg(U + j * q + c), a0);
                    a1 = fmaf(d, __ldg(U + (j + 1) * q + c), a1);
                    a2 = fmaf(d, __ldg(U + (j + 2) * q + c), a2);
                    a3 = fmaf(d, __ldg(U + (j + 3) * q + c), a3);
                }
            }
            if (snap) {
                const float4 sv = snap[e4];
                a0 += sv.x;
                a1 += sv.y;
                a2 += sv.z;
                a3 += sv.w;
            }
            out[e4] = make_float4(a0, a1, a2, a3);
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
    const int per_row = p.n * p.n / 4;
    const int64_t rpi = per_row >= 256 ? 1 : 256 / per_row;
    const int64_t need = (rows + rpi - 1) / rpi;
    const int64_t blocks = need < (int64_t)sms * 8 ? need : (int64_t)sms * 8;
    const size_t staged = sizeof(float) * (size_t)(u_hs == 0 ? 1 : p.H) * (size_t)p.n * q;
    if (staged <= 48 * 1024)
        k_readout_grad<true><<<(unsigned)blocks, 256, staged, s>>>(p.B, p.L, p.H, p.n, q, u_hs, u, d_o, every, d_snap,
                                                                   dS);
    else
        k_readout_grad<false><<<(unsigned)blocks, 256, 0, s>>>(p.B, p.L, p.H, p.n, q, u_hs, u, d_o, every, d_snap, dS);
    return cudaGetLastError();
}

}  // namespace mru
