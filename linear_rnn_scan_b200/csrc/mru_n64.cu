// mru_n64.cu -- n = 64 determinant-corrected scan with the readout
// (o_t = S_t U, snapshots), chunk phase on the tensor cores.
//
// One CTA of 4 warps per chain (b, h, chunk); warp w owns rows 16w..16w+15
// of the 64 x 64 state Q = P - I, held in mma accumulator registers.  Per
// token:
//   * the slice is copied to shared memory (cp.async),
//   * the determinant scale c = |det(I + alpha M)|^(-1/64) comes from an LU
//     of E = alpha M in identity-split form (pivots 1 + delta_k), register
//     blocked: thread (br, bc) owns rows 4br..4br+3, columns 8bc..8bc+7; the
//     pivot row and column are exchanged through shared memory, one barrier
//     per step; |det| = prod (1 + delta_k) in fp32, c - 1 by log1p and expm1.
//     A pivot below 1/2 in magnitude sends the token to a partially pivoted
//     LU in shared memory,
//   * Q_t = Q_{t-1} + (F_t + Q_{t-1} F_t) with F = c alpha M + (c - 1) I,
//     the product on mma.sync m16n8k8 tf32 with fp32 accumulation (the
//     workload's tf32 arithmetic; the identity split keeps the implicit 1 out
//     of the tf32 operands); the contraction index is permuted so that the
//     accumulator tile j is the A fragment of k-tile j,
//   * V_t = Q_t U (the readout of the local prefix, U the head's q query
//     columns) is written where o_t goes, and Q_t where a snapshot is due;
//     the chunk total goes to the workspace.
// The carry scan and the fix-up o_t = C U + C V_t are the generic kernels.
#include "mru_internal.cuh"

namespace mru {
namespace n64 {
namespace {

constexpr int N = 64;
constexpr int NN = N * N;
constexpr int ROWW = 68;             // padded shared-memory row stride in words
constexpr int THREADS = 128;

struct Smem {
    float x[N * ROWW];               // 17,408 bytes: the token's slice
    float prow[2][N];                // pivot row, double-buffered by step parity
    float pcol[2][N];                // pivot column
    float ut[N * N];                 // the head's query columns U, transposed: ut[c][j] = U[j][c]
    double dsum;                     // pivoted fallback: log|det|
    int flag;
    int piv;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::); }

__device__ __forceinline__ uint32_t to_tf32(float v)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// |det(I + alpha M)| (ok == true) by the register-blocked identity-split
// LU; ok == false when a pivot is below 1/2 in magnitude.  All threads call.
// Thread (br, bc) updates its whole 4 x 8 block at every step where the block
// reaches below and right of the pivot: entries in eliminated rows or columns
// are never read again, so they need no masking.
__device__ float absdet_near_identity(Smem& sm, float alpha, bool& ok)
{
    const int t = threadIdx.x, br = t >> 3, bc = t & 7;
    float e[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float4* row = reinterpret_cast<const float4*>(sm.x + (4 * br + r) * ROWW + 8 * bc);
        const float4 v0 = row[0], v1 = row[1];
        e[r][0] = alpha * v0.x; e[r][1] = alpha * v0.y; e[r][2] = alpha * v0.z; e[r][3] = alpha * v0.w;
        e[r][4] = alpha * v1.x; e[r][5] = alpha * v1.y; e[r][6] = alpha * v1.z; e[r][7] = alpha * v1.w;
    }
    float prod = 1.0f;
    bool good = true;
    // k = k0 + kk with kk unrolled, so that the register slots selected by
    // k & 3 and k & 7 are known at compile time (no local-memory arrays)
    for (int k0 = 0; k0 < N; k0 += 8) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int k = k0 + kk;
            const int par = kk & 1;
            if (br == (k >> 2)) {
                float4* pr = reinterpret_cast<float4*>(sm.prow[par] + 8 * bc);
                pr[0] = make_float4(e[kk & 3][0], e[kk & 3][1], e[kk & 3][2], e[kk & 3][3]);
                pr[1] = make_float4(e[kk & 3][4], e[kk & 3][5], e[kk & 3][6], e[kk & 3][7]);
            }
            if (bc == (k >> 3))
                *reinterpret_cast<float4*>(sm.pcol[par] + 4 * br) = make_float4(e[0][kk], e[1][kk], e[2][kk], e[3][kk]);
            __syncthreads();
            const float pk = 1.0f + sm.prow[par][k];
            if (!(fabsf(pk) >= 0.5f)) good = false;
            prod *= pk;
            if (4 * br + 3 > k && 8 * bc + 7 > k) {
                float rk;
                asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(rk) : "f"(pk));
                const float4 lc = *reinterpret_cast<const float4*>(sm.pcol[par] + 4 * br);
                const float4 p0 = *reinterpret_cast<const float4*>(sm.prow[par] + 8 * bc);
                const float4 p1 = *reinterpret_cast<const float4*>(sm.prow[par] + 8 * bc + 4);
                const float l[4] = {lc.x * rk, lc.y * rk, lc.z * rk, lc.w * rk};
                const float pr[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int c = 0; c < 8; ++c) e[r][c] = fmaf(-l[r], pr[c], e[r][c]);
            }
        }
    }
    ok = good;
    return fabsf(prod);
}

// log|det(W)|, W = add_identity I + alpha M, by LU with partial pivoting on
// a copy in shared memory (the slice buffer is overwritten; it is reloaded
// afterwards).  Returns NaN when a pivot column is zero.
__device__ double logdet_pivoted(Smem& sm, float alpha, int add_identity)
{
    const int t = threadIdx.x;
    float* W = sm.x;
    for (int e = t; e < NN; e += THREADS) {
        const int i = e / N, j = e % N;
        float v = alpha * W[i * ROWW + j];
        if (add_identity && i == j) v += 1.0f;
        W[i * ROWW + j] = v;
    }
    if (t == 0) { sm.dsum = 0.0; sm.flag = 0; }
    __syncthreads();
    for (int k = 0; k < N; ++k) {
        if (t < 32) {
            float best = -1.0f;
            int bi = k;
            for (int i = k + t; i < N; i += 32) {
                const float a = fabsf(W[i * ROWW + k]);
                if (a > best) { best = a; bi = i; }
            }
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_down_sync(0xffffffffu, best, o);
                const int oi = __shfl_down_sync(0xffffffffu, bi, o);
                if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            if (t == 0) {
                sm.piv = bi;
                if (!(best > 0.0f)) sm.flag = 1;
            }
        }
        __syncthreads();
        const int piv = sm.piv;
        if (piv != k)
            for (int j = t; j < N; j += THREADS) {
                const float a = W[k * ROWW + j];
                W[k * ROWW + j] = W[piv * ROWW + j];
                W[piv * ROWW + j] = a;
            }
        __syncthreads();
        const float pk = W[k * ROWW + k];
        if (t == 0) sm.dsum += log(fabs((double)pk));
        const float r = (pk != 0.0f) ? 1.0f / pk : 0.0f;
        const int m = N - k - 1;
        for (int idx = t; idx < m * m; idx += THREADS) {
            const int i = k + 1 + idx / m, j = k + 1 + idx % m;
            W[i * ROWW + j] = fmaf(-W[i * ROWW + k] * r, W[k * ROWW + j], W[i * ROWW + j]);
        }
        __syncthreads();
    }
    const double ld = sm.dsum;
    const bool bad = sm.flag != 0;
    __syncthreads();
    return bad ? __longlong_as_double(0x7ff8000000000000ll) : ld;
}

__device__ __forceinline__ void load_slice(Smem& sm, const float* src)
{
    for (int g = threadIdx.x; g < NN / 4; g += THREADS) {
        const int row = g >> 4, c4 = g & 15;
        cp_async16(sm.x + row * ROWW + 4 * c4, src + row * N + 4 * c4);
    }
    cp_async_wait_all();
    __syncthreads();
}

__global__ void __launch_bounds__(THREADS, 4)
k64_chunk_readout(KParams p, const float* __restrict__ x, const float* __restrict__ u, int64_t snap_every,
                  float* __restrict__ o_out, float* __restrict__ snaps, float* __restrict__ totals,
                  uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const int64_t chain = blockIdx.x;                // (b*H + h)*K + k, like the generic kernels
    const int64_t k = chain % p.K, bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    const int64_t tok = p.H * NN;
    const float* xb = x + (b * p.L * p.H + h) * NN;

    const int rq = p.rq;
    for (int e = tid; e < N * rq; e += THREADS) {
        const int j = e / rq, c = e - j * rq;
        sm.ut[c * N + j] = u[h * p.u_hs + e];
    }
    __syncthreads();
    const int r0 = 16 * warp;                        // this warp's rows
    float Qd[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) Qd[nt][i] = 0.0f;

    for (int64_t t = t0; t < t1; ++t) {
        const float* src = xb + t * tok;
        load_slice(sm, src);
        // ---- determinant scale ----
        float ca = p.alpha, dv = p.add_identity ? 0.0f : -1.0f;
        if (p.mode == MRU_MODE_DETNORM) {
            // near the identity: |det| = prod (1 + delta_k) in fp32 (64
            // factors near 1, relative error about 2e-7), c - 1 =
            // expm1(-log1p(|det| - 1) / 64); otherwise the pivoted LU's fp64 sum
            float cm1 = 0.0f;
            bool ok = p.add_identity != 0;
            if (ok) cm1 = expm1f(-log1pf(absdet_near_identity(sm, p.alpha, ok) - 1.0f) * (1.0f / N));
            __syncthreads();
            const bool retry = __syncthreads_or(!ok);
            bool bad = false;
            if (retry) {
                const double ld = logdet_pivoted(sm, p.alpha, p.add_identity);
                load_slice(sm, src);                 // the fallback overwrote the slice
                bad = !isfinite(ld);
                cm1 = (float)expm1(-ld / N);
            }
            const float c = 1.0f + cm1;
            if (bad || !isfinite(cm1) || !(c > 0.0f)) {
                if (tid == 0) atomicOr(status, STATUS_SINGULAR);
                ca = 0.0f;
                dv = 0.0f;
            } else {
                ca = c * p.alpha;
                dv = p.add_identity ? cm1 : -1.0f;
            }
        }
        // ---- Q_t = Q + (F + Q F), 1xTF32 ----
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
#pragma unroll
        for (int kt = 0; kt < 8; ++kt) {
            uint32_t a[4];
            a[0] = to_tf32(Qd[kt][0]);
            a[1] = to_tf32(Qd[kt][2]);
            a[2] = to_tf32(Qd[kt][1]);
            a[3] = to_tf32(Qd[kt][3]);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                // B fragment, contraction index permuted: slot q <-> row 8kt + 2q
                const float* base = sm.x + (8 * kt + 2 * q) * ROWW + 8 * nt + g;
                float v0 = ca * base[0], v1 = ca * base[ROWW];
                if (kt == nt) {
                    if (g == 2 * q) v0 += dv;
                    if (g == 2 * q + 1) v1 += dv;
                }
                mma_tf32(acc[nt], a, to_tf32(v0), to_tf32(v1));
            }
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                const float2 xv = *reinterpret_cast<const float2*>(sm.x + row * ROWW + col);
                float f0 = ca * xv.x, f1 = ca * xv.y;
                if (row == col) f0 += dv;
                if (row == col + 1) f1 += dv;
                Qd[nt][2 * h8] += f0 + acc[nt][2 * h8];
                Qd[nt][2 * h8 + 1] += f1 + acc[nt][2 * h8 + 1];
            }
        // ---- readout of the local prefix: V_t = Q_t U (rq columns; the loop
        // bound is uniform over the CTA, so every lane reaches the shuffles) ----
        const int64_t row_bth = (b * p.L + t) * p.H + h;
        for (int c = 0; c < rq; ++c) {
            float ur[8][2];                          // U[:, c] at this lane's columns 8 nt + 2 q, + 1
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const float2 v = *reinterpret_cast<const float2*>(sm.ut + c * N + 8 * nt + 2 * q);
                ur[nt][0] = v.x;
                ur[nt][1] = v.y;
            }
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                float s = 0.0f;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    s = fmaf(Qd[nt][2 * h8], ur[nt][0], s);
                    s = fmaf(Qd[nt][2 * h8 + 1], ur[nt][1], s);
                }
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                if (q == 0) o_out[(row_bth * N + r0 + g + 8 * h8) * rq + c] = s;
            }
        }
        if (snap_every > 0 && ((t + 1) % snap_every) == 0) {
            const int64_t srow = (b * (p.L / snap_every) + (t + 1) / snap_every - 1) * p.H + h;
            float* sp = snaps + srow * NN;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8)
                    *reinterpret_cast<float2*>(sp + (r0 + g + 8 * h8) * N + 8 * nt + 2 * q) =
                        make_float2(Qd[nt][2 * h8], Qd[nt][2 * h8 + 1]);
        }
        __syncthreads();                             // slice buffer reused by the next token
    }
    float* tot = totals + chain * NN;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8)
            *reinterpret_cast<float2*>(tot + (r0 + g + 8 * h8) * N + 8 * nt + 2 * q) =
                make_float2(Qd[nt][2 * h8], Qd[nt][2 * h8 + 1]);
}

}  // namespace

bool supports(const KParams& p, bool readout)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_F32 && readout && p.K > 1 &&
           (p.mode == MRU_MODE_DETNORM || p.mode == MRU_MODE_RESHAPE) &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_TF32);
}

cudaError_t launch_chunk_readout(const KParams& p, const float* x, const float* u, int64_t snap_every,
                                 float* o_out, float* snaps, float* totals, uint32_t* status, cudaStream_t s)
{
    const int64_t chains = p.B * p.H * p.K;
    const size_t sm = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(k64_chunk_readout, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k64_chunk_readout<<<(unsigned)chains, THREADS, sm, s>>>(p, x, u, snap_every, o_out, snaps, totals, status);
    return cudaGetLastError();
}

}  // namespace n64
}  // namespace mru
