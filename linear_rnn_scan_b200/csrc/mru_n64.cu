// mru_n64.cu -- n = 64 determinant-corrected scan with the readout
// (o_t = S_t U, snapshots), chunk phase on the tensor cores.
//
// One CTA of 4 warps per chain (b, h, chunk); warp w owns rows 16w..16w+15
// of the 64 x 64 state Q = P - I, held in mma accumulator registers.  Per
// token:
//   * the slice arrives in one of two shared-memory buffers (cp.async; the
//     next token's copy is in flight meanwhile),
//   * the determinant scale c = |det(I + alpha M)|^(-1/64): from the trace
//     series of log det (M2 = M M and M3 = M2 M on the tensor cores in bf16,
//     traces and norms summed over the CTA, a remainder bound deciding), or
//     where the bound does not certify it from an LU of E = alpha M in
//     identity-split form (register blocked, one barrier per step), and
//     far from the identity from a partially pivoted LU in shared memory,
//   * Q_t = Q_{t-1} + (F_t + Q_{t-1} F_t) with F = c alpha M + (c - 1) I,
//     Q F formed as c alpha (Q M) + (c - 1) Q, the product on mma.sync
//     m16n8k8 tf32 with fp32 accumulation (the workload's tf32 arithmetic;
//     the identity split keeps the implicit 1 out of the tf32 operands); the
//     contraction index is permuted so that the accumulator tile j is the A
//     fragment of k-tile j,
//   * V_t = Q_t U (the readout of the local prefix, U the head's q query
//     columns) is written where o_t goes, and Q_t where a snapshot is due;
//     the chunk total goes to the workspace.
// The carry scan is the generic one; the fix-up o_t = C U + C V_t (and the
// snapshots C + C Q_t) is k64_fixup below, on the tensor cores.
//
// k64_chunk_readout_tc (opt-in, MRU_N64_TCGEN05=1) runs the same chunk phase
// with the three products on tcgen05 and tensor memory; see its section.
#include <stdlib.h>

#include "mru_internal.cuh"

namespace mru {
namespace n64 {
namespace {

constexpr int N = 64;
constexpr int NN = N * N;
constexpr int ROWW = 68;             // padded shared-memory row stride in words
constexpr int THREADS = 128;

struct Smem {
    float x[2][N * ROWW];            // 2 x 17,408 bytes: this token's slice and the next one's
    float prow[2][N];                // pivot row, double-buffered by step parity
    float pcol[2][N];                // pivot column
    float ut[N * N];                 // the head's query columns U, transposed: ut[c][j] = U[j][c]
    float red[4][8];                 // per-warp partial traces and norms
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

// v rounded to the nearest tf32, ties away from zero (the magnitude bits plus
// half a unit of the 10th mantissa bit, then truncated): two integer
// operations on the ALU pipe, the same value cvt.rna.tf32.f32 gives for
// finite v.
__device__ __forceinline__ uint32_t to_tf32(float v) { return (__float_as_uint(v) + 0x1000u) & 0xffffe000u; }

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
__device__ float absdet_near_identity(Smem& sm, const float* xs, float alpha, bool& ok)
{
    const int t = threadIdx.x, br = t >> 3, bc = t & 7;
    float e[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float4* row = reinterpret_cast<const float4*>(xs + (4 * br + r) * ROWW + 8 * bc);
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
__device__ double logdet_pivoted(Smem& sm, float* W, float alpha, int add_identity)
{
    const int t = threadIdx.x;
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

// D += A B, m16n8k16, bf16 operands, fp32 accumulate (the determinant's series).
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 pair (lo_elem in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// bf16 B fragment of the raw slice M for k-tile kt (16 rows) and column
// tile nt: b0 = M[16 kt + 2 q, + 1][8 nt + g], b1 the same 8 rows lower.
__device__ __forceinline__ void frag_m16(const float* xs, int kt, int nt, int g, int q, uint32_t& b0, uint32_t& b1)
{
    const float* base = xs + (16 * kt + 2 * q) * ROWW + 8 * nt + g;
    b0 = pack_bf16(base[0], base[ROWW]);
    b1 = pack_bf16(base[8 * ROWW], base[9 * ROWW]);
}

// Copies a token's slice into a slice buffer (cp.async, committed as one group).
__device__ __forceinline__ void issue_slice(float* xs, const float* src)
{
    for (int g = threadIdx.x; g < NN / 4; g += THREADS) {
        const int row = g >> 4, c4 = g & 15;
        cp_async16(xs + row * ROWW + 4 * c4, src + row * N + 4 * c4);
    }
    asm volatile("cp.async.commit_group;\n" ::);
}

// Plain reload of a slice (after the pivoted fallback has overwritten it).
__device__ __forceinline__ void reload_slice(float* xs, const float* src)
{
    for (int g = threadIdx.x; g < NN / 4; g += THREADS) {
        const int row = g >> 4, c4 = g & 15;
        *reinterpret_cast<float4*>(xs + row * ROWW + 4 * c4) = *reinterpret_cast<const float4*>(src + row * N + 4 * c4);
    }
    __syncthreads();
}

// B fragment of the raw slice M for k-tile kt and column tile nt, the
// contraction index permuted as for the accumulator-resident A operands
// (slot q <-> row 8 kt + 2 q, slot q + 4 <-> row 8 kt + 2 q + 1).
__device__ __forceinline__ void frag_m(const float* xs, int kt, int nt, int g, int q, uint32_t& b0, uint32_t& b1)
{
    const float* base = xs + (8 * kt + 2 * q) * ROWW + 8 * nt + g;
    b0 = to_tf32(base[0]);
    b1 = to_tf32(base[ROWW]);
}

// Sum over the warp, the same value in every lane.
__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
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

    // the determinant scale by the trace series (see series_logdet) where its
    // certificate holds; the near-identity LU otherwise
    const bool detnorm = p.mode == MRU_MODE_DETNORM;
    const bool series = detnorm && p.add_identity != 0;
    issue_slice(sm.x[0], xb + t0 * tok);
    for (int64_t t = t0; t < t1; ++t) {
        const int cur = (int)((t - t0) & 1);
        float* xs = sm.x[cur];
        if (t + 1 < t1) issue_slice(sm.x[cur ^ 1], xb + (t + 1) * tok);
        else asm volatile("cp.async.commit_group;\n" ::);
        asm volatile("cp.async.wait_group 1;\n" ::);
        __syncthreads();

        // ---- for the series: M2 = M M over this warp's rows ----
        float M2[8][4];
        if (series) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) M2[nt][i] = 0.0f;
#pragma unroll
            for (int kt = 0; kt < 4; ++kt) {                // bf16 m16n8k16: 16 contraction rows a step
                uint32_t am[4];
                const float2 m0 = *reinterpret_cast<const float2*>(xs + (r0 + g) * ROWW + 16 * kt + 2 * q);
                const float2 m1 = *reinterpret_cast<const float2*>(xs + (r0 + g + 8) * ROWW + 16 * kt + 2 * q);
                const float2 m2 = *reinterpret_cast<const float2*>(xs + (r0 + g) * ROWW + 16 * kt + 8 + 2 * q);
                const float2 m3 = *reinterpret_cast<const float2*>(xs + (r0 + g + 8) * ROWW + 16 * kt + 8 + 2 * q);
                am[0] = pack_bf16(m0.x, m0.y);
                am[1] = pack_bf16(m1.x, m1.y);
                am[2] = pack_bf16(m2.x, m2.y);
                am[3] = pack_bf16(m3.x, m3.y);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    uint32_t b0, b1;
                    frag_m16(xs, kt, nt, g, q, b0, b1);
                    mma_bf16(M2[nt], am, b0, b1);
                }
            }
        }

        // ---- determinant scale ----
        float ca = p.alpha, dv = p.add_identity ? 0.0f : -1.0f;
        if (detnorm) {
            bool ok = false;
            float cm1 = 0.0f;
            if (series) {
                // log det(I + E), E = alpha M, by its trace series
                //   tr E - tr E^2 / 2 + tr E^3 / 3 - tr E^4 / 4 + R,
                // tr E^k = <E^(k-1), E^T> from M2 = M M and M3 = M2 M (bf16
                // products on the tensor cores, m16n8k16).  Since tr E^k = <E^(k-3), (E^3)^T>
                // and |E^m|_F <= |E^2|_F |E|_F^(m-2),
                //   |R| <= |E^3|_F |E^2|_F / (5 (1 - |E|_F))   (|E|_F < 1),
                // the series is taken when that bound is at most 1e-6 (the scale
                // c = exp(-log det / 64) then good to 1.6e-8; the bf16 rounding of
                // the products' operands adds about 1e-7 to log det at the
                // workload's alpha).
                float tr1 = 0.0f, tr2 = 0.0f, tr3 = 0.0f, tr4 = 0.0f, n1 = 0.0f, n2 = 0.0f, n3 = 0.0f;
                if (lane < 16) tr1 = xs[(r0 + lane) * ROWW + r0 + lane];
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                        const float2 mv = *reinterpret_cast<const float2*>(xs + row * ROWW + col);
                        const float mt0 = xs[col * ROWW + row], mt1 = xs[(col + 1) * ROWW + row];   // M^T here
                        tr2 = fmaf(mv.x, mt0, fmaf(mv.y, mt1, tr2));
                        tr3 = fmaf(M2[nt][2 * h8], mt0, fmaf(M2[nt][2 * h8 + 1], mt1, tr3));
                        n1 = fmaf(mv.x, mv.x, fmaf(mv.y, mv.y, n1));
                        n2 = fmaf(M2[nt][2 * h8], M2[nt][2 * h8], fmaf(M2[nt][2 * h8 + 1], M2[nt][2 * h8 + 1], n2));
                    }
                // M3 = M2 M, four column tiles at a time
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float M3[4][4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int i = 0; i < 4; ++i) M3[j][i] = 0.0f;
#pragma unroll
                    for (int kt = 0; kt < 4; ++kt) {
                        // accumulator tiles 2 kt, 2 kt + 1 are the bf16 A fragment of k-tile kt
                        uint32_t a[4];
                        a[0] = pack_bf16(M2[2 * kt][0], M2[2 * kt][1]);
                        a[1] = pack_bf16(M2[2 * kt][2], M2[2 * kt][3]);
                        a[2] = pack_bf16(M2[2 * kt + 1][0], M2[2 * kt + 1][1]);
                        a[3] = pack_bf16(M2[2 * kt + 1][2], M2[2 * kt + 1][3]);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t b0, b1;
                            frag_m16(xs, kt, 4 * hh + j, g, q, b0, b1);
                            mma_bf16(M3[j], a, b0, b1);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int h8 = 0; h8 < 2; ++h8) {
                            const int row = r0 + g + 8 * h8, col = 8 * (4 * hh + j) + 2 * q;
                            const float mt0 = xs[col * ROWW + row], mt1 = xs[(col + 1) * ROWW + row];
                            tr4 = fmaf(M3[j][2 * h8], mt0, fmaf(M3[j][2 * h8 + 1], mt1, tr4));
                            n3 = fmaf(M3[j][2 * h8], M3[j][2 * h8], fmaf(M3[j][2 * h8 + 1], M3[j][2 * h8 + 1], n3));
                        }
                }
                tr1 = warp_sum(tr1);
                tr2 = warp_sum(tr2);
                tr3 = warp_sum(tr3);
                tr4 = warp_sum(tr4);
                n1 = warp_sum(n1);
                n2 = warp_sum(n2);
                n3 = warp_sum(n3);
                if (lane == 0) {
                    float* rd = sm.red[warp];
                    rd[0] = tr1; rd[1] = tr2; rd[2] = tr3; rd[3] = tr4; rd[4] = n1; rd[5] = n2; rd[6] = n3;
                }
                __syncthreads();
                float v[7];
#pragma unroll
                for (int i = 0; i < 7; ++i) v[i] = (sm.red[0][i] + sm.red[1][i]) + (sm.red[2][i] + sm.red[3][i]);
                const float a = p.alpha, a2 = a * a;
                const float ld = a * v[0] - a2 * (0.5f * v[1]) + a2 * a * (v[2] * (1.0f / 3.0f)) -
                                 a2 * a2 * (0.25f * v[3]);
                const float fe = a * sqrtf(v[4]), fe2 = a2 * sqrtf(v[5]), fe3 = a2 * a * sqrtf(v[6]);
                const float bound = fe3 * fe2 / (5.0f * (1.0f - fe));
                ok = fe < 1.0f && bound <= 1e-6f;      // false for non-finite inputs too
                if (ok) cm1 = expm1f(-ld * (1.0f / N));
            }
            if (!ok) {
                // near the identity: |det| = prod (1 + delta_k) in fp32 (64
                // factors near 1, relative error about 2e-7), c - 1 =
                // expm1(-log1p(|det| - 1) / 64); otherwise the pivoted LU's fp64 sum
                bool near = p.add_identity != 0;
                if (near) cm1 = expm1f(-log1pf(absdet_near_identity(sm, xs, p.alpha, near) - 1.0f) * (1.0f / N));
                __syncthreads();
                const bool retry = __syncthreads_or(!near);
                bool bad = false;
                if (retry) {
                    const double ld = logdet_pivoted(sm, xs, p.alpha, p.add_identity);
                    reload_slice(xs, xb + t * tok);      // the fallback overwrote the slice
                    bad = !isfinite(ld);
                    cm1 = (float)expm1(-ld / N);
                }
                ok = !bad;
            }
            const float c = 1.0f + cm1;
            if (!ok || !isfinite(cm1) || !(c > 0.0f)) {
                if (tid == 0) atomicOr(status, STATUS_SINGULAR);
                ca = 0.0f;
                dv = 0.0f;
            } else {
                ca = c * p.alpha;
                dv = p.add_identity ? cm1 : -1.0f;
            }
        }
        // ---- Q_t = Q + (F + Q F), Q F = ca Q M + dv Q, F = ca M + dv I ----
        float P[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) P[nt][i] = 0.0f;
#pragma unroll
        for (int kt = 0; kt < 8; ++kt) {
            uint32_t aq[4];
            aq[0] = to_tf32(Qd[kt][0]);
            aq[1] = to_tf32(Qd[kt][2]);
            aq[2] = to_tf32(Qd[kt][1]);
            aq[3] = to_tf32(Qd[kt][3]);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                uint32_t b0, b1;
                frag_m(xs, kt, nt, g, q, b0, b1);
                mma_tf32(P[nt], aq, b0, b1);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                const float2 xv = *reinterpret_cast<const float2*>(xs + row * ROWW + col);
                float f0 = ca * xv.x, f1 = ca * xv.y;
                if (row == col) f0 += dv;
                if (row == col + 1) f1 += dv;
                const float q0 = fmaf(ca, P[nt][2 * h8], dv * Qd[nt][2 * h8]);
                const float q1 = fmaf(ca, P[nt][2 * h8 + 1], dv * Qd[nt][2 * h8 + 1]);
                Qd[nt][2 * h8] += f0 + q0;
                Qd[nt][2 * h8 + 1] += f1 + q1;
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

// ---- fix-up of the readout on the tensor cores ------------------------------
//
// Per chain (one CTA of 4 warps, warp w owns rows 16 w .. 16 w + 15 of the
// chain's carry C): o_t = C U + C V_t for every token of the chunk (V_t the
// chunk kernel's local readout, written where o_t goes), as products of C
// with blocks of the matrix [V_t0 .. V_t1-1] (64 rows, q columns per token)
// staged in shared memory two blocks at a time; C U once per chain; and the
// snapshots S_t = C + C Q_t.  tf32 mma.sync with fp32 accumulation, the
// chunk kernel's arithmetic.

constexpr int FX_COLS = 64;                      // columns of a staged block
constexpr int FX_BUF = N * (N + 4);              // floats per staging buffer (fits a padded 64 x 64 Q_t too)

// acc = C W for column tile nt of a staged block: C in A fragments ca (plain
// contraction order), W column col at offset boff of the buffer, entries
// `ld` words apart.
__device__ __forceinline__ void fx_tile(const uint32_t (&ca)[8][4], const float* buf, int boff, int ld, int qq,
                                        float (&acc)[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt)
        mma_tf32(acc, ca[kt], to_tf32(buf[boff + (8 * kt + qq) * ld]), to_tf32(buf[boff + (8 * kt + qq + 4) * ld]));
}

__global__ void __launch_bounds__(THREADS, 4)
k64_fixup(KParams p, const float* __restrict__ carry, const float* __restrict__ u, int64_t snap_every,
          float* __restrict__ o_out, float* __restrict__ snaps)
{
    extern __shared__ __align__(16) float fsm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, qq = lane & 3;
    const int q = p.rq, nq = N * q;                         // q = 0: snapshots only (full states)
    const int tpb = q > 0 && FX_COLS / q > 0 ? FX_COLS / q : 1;   // tokens per staged block
    const int TS = nq + 4;                                  // padded words per staged token
    float* sCU = fsm + 2 * FX_BUF;                          // C U, [64][q]
    const int64_t chain = blockIdx.x;
    const int64_t k = chain % p.K, bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    const int r0 = 16 * warp;
    const float* C = carry + chain * NN;
    uint32_t ca[8][4];
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
        ca[kt][0] = to_tf32(C[(r0 + g) * N + 8 * kt + qq]);
        ca[kt][1] = to_tf32(C[(r0 + g + 8) * N + 8 * kt + qq]);
        ca[kt][2] = to_tf32(C[(r0 + g) * N + 8 * kt + qq + 4]);
        ca[kt][3] = to_tf32(C[(r0 + g + 8) * N + 8 * kt + qq + 4]);
    }
    auto issue = [&](float* dst, int64_t tb) {          // the block of tokens tb .. (cp.async)
        const int ntok = (int)((t1 - tb < tpb) ? t1 - tb : tpb);
        const int gran = nq / 4;                          // 16-byte granules a token
        for (int i = tid; i < ntok * gran; i += THREADS) {
            const int tt = i / gran, gg = i - tt * gran;
            cp_async16(dst + tt * TS + 4 * gg, o_out + ((b * p.L + tb + tt) * p.H + h) * nq + 4 * gg);
        }
        asm volatile("cp.async.commit_group;\n" ::);
    };
    if (q > 0 && t0 < t1) issue(fsm + FX_BUF, t0);
    // C U (U staged as one token of the block layout in the first buffer)
    for (int e = tid; e < nq; e += THREADS) fsm[e] = u[h * p.u_hs + e];
    __syncthreads();
    for (int nt = 0; nt * 8 < q; ++nt) {
        const int cb = 8 * nt + g;
        float acc[4];
        fx_tile(ca, fsm, cb < q ? cb : 0, q, qq, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = r0 + g + 8 * (i >> 1), c = 8 * nt + 2 * qq + (i & 1);
            if (c < q) sCU[row * q + c] = acc[i];
        }
    }
    __syncthreads();
    // the chunk's tokens, a block at a time: o = C U + C V
    int cur = 1;
    for (int64_t tb = t0; q > 0 && tb < t1; tb += tpb) {
        const int64_t tn = tb + tpb;
        if (tn < t1) issue(fsm + (cur ^ 1) * FX_BUF, tn);
        else asm volatile("cp.async.commit_group;\n" ::);
        asm volatile("cp.async.wait_group 1;\n" ::);
        __syncthreads();
        const float* w = fsm + cur * FX_BUF;
        const int ncol = (int)((t1 - tb < tpb) ? t1 - tb : tpb) * q;
        for (int nt = 0; nt * 8 < ncol; ++nt) {
            const int cb = 8 * nt + g;
            const int boff = cb < ncol ? (cb / q) * TS + cb % q : 0;
            float acc[4];
            fx_tile(ca, w, boff, q, qq, acc);
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                const int col = 8 * nt + 2 * qq + s2;
                if (col < ncol) {
                    const int tt = col / q, c = col - tt * q;
                    float* dst = o_out + ((b * p.L + tb + tt) * p.H + h) * nq;
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int row = r0 + g + 8 * h8;
                        dst[row * q + c] = sCU[row * q + c] + acc[2 * h8 + s2];
                    }
                }
            }
        }
        __syncthreads();
        cur ^= 1;
    }
    // snapshots: S_t = C + C Q_t, Q_t staged with rows padded to N + 4 words
    if (snap_every > 0) {
        const int64_t first = ((t0 + snap_every) / snap_every) * snap_every;   // 1-based
        for (int64_t t1b = first; t1b <= t1; t1b += snap_every) {
            float* sp = snaps + ((b * (p.L / snap_every) + t1b / snap_every - 1) * p.H + h) * NN;
            for (int e = tid; e < NN / 4; e += THREADS) {
                const int row = e >> 4, c4 = e & 15;
                *reinterpret_cast<float4*>(fsm + row * (N + 4) + 4 * c4) =
                    *reinterpret_cast<const float4*>(sp + row * N + 4 * c4);
            }
            __syncthreads();
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                float acc[4];
                fx_tile(ca, fsm, 8 * nt + g, N + 4, qq, acc);
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * qq;
                    const float2 cv = *reinterpret_cast<const float2*>(C + row * N + col);
                    *reinterpret_cast<float2*>(sp + row * N + col) =
                        make_float2(cv.x + acc[2 * h8], cv.y + acc[2 * h8 + 1]);
                }
            }
            __syncthreads();
        }
    }
}

// ---- the chunk phase on tcgen05 (opt-in: MRU_N64_TCGEN05=1) -----------------
//
// The same computation with the three 64 x 64 x 64 products on the
// fifth-generation tensor cores: the slice in the block layout the tensor
// cores read (core matrices of 8 rows x 16 bytes), M^T rounded to tf32 as the
// B operand (K-major) of every product, Q_{t-1} or M^2 as the A operand; one
// thread issues tcgen05.mma kind::tf32 (M = 64, N = 64, eight K = 8 steps)
// into tensor memory and commits to an mbarrier (bounded wait); each warp
// reads its 16 rows back with tcgen05.ld 16x256b, which hands every thread
// the mma accumulator fragment of its rows.  Correct and tested, but slower
// than the mma.sync kernel above on B200: per token and CTA the products'
// waits are a sixth of the time, the rest is the element-wise work around
// them (the transposition of M, the trace sums, the update and the readout)
// and seven CTA barriers, with three CTAs per SM (shared memory) instead of
// four.
namespace tc {

constexpr int CSB = 1024;            // block layout: bytes between column groups (8-row groups are 128 B apart)

// Byte offset of element (r, c) of a 64 x 64 fp32 matrix in the block layout
// (no swizzle): core matrices of 8 rows x 4 columns (16 bytes a row) stored
// contiguously, 8-row groups 128 bytes apart, 4-column groups CSB apart.  As
// a K-major tensor-core operand (rows = M or N, columns = K) its descriptor
// has leading byte offset CSB (the two K halves of a K = 8 step) and stride
// byte offset 128 (the 8-row groups).
__host__ __device__ __forceinline__ int boff(int r, int c)
{
    return (r >> 3) * 128 + (c >> 2) * CSB + (r & 7) * 16 + (c & 3) * 4;
}

struct Smem {
    float mb[2][NN];                 // slices M (block layout, as loaded): this token's and the next one's
    float mt[NN];                    // M^T rounded to tf32 (block layout): the B operand of every product
    float qa[NN];                    // the A operand: Q_{t-1} or M^2, rounded to tf32 (block layout)
    float prow[2][N];                // near-identity LU: pivot row, double-buffered by step parity
    float pcol[2][N];                // pivot column
    float red[4][8];                 // per-warp partial traces and norms
    double dsum;                     // pivoted fallback: log|det|
    unsigned long long mbar;         // tensor-core completion barrier
    int flag;
    int piv;
    uint32_t tmem;                   // tensor-memory base address (128 columns)
    // followed by U transposed, [rq][N] floats
};
static_assert(sizeof(float) * N * ROWW <= 2 * sizeof(float) * NN, "pivoted LU scratch fits mt and qa");

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }


__device__ __forceinline__ float round_tf32(float v) { return __uint_as_float(to_tf32(v)); }


// ---- fifth-generation tensor cores (tcgen05) --------------------------------

// Shared-memory descriptor of a K-major operand in the block layout: start
// address >> 4 (bits 0-13), leading byte offset >> 4 (bits 16-29), stride
// byte offset >> 4 (bits 32-45), descriptor version 1 (bit 46), no swizzle
// (bits 61-63 zero).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3fffu) | ((uint64_t)(CSB >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
           (1ull << 46);
}

// Instruction descriptor of kind::tf32: fp32 accumulator (bits 4-5 = 1),
// A and B tf32 (bits 7-9, 10-12 = 2), both K-major (bits 15, 16 = 0),
// N = 64 (bits 17-22 = N / 8), M = 64 (bits 24-28 = M / 16).
constexpr uint32_t kIdescTf32 = (1u << 4) | (2u << 7) | (2u << 10) | ((64u / 8) << 17) | ((64u / 16) << 24);

// D (tensor memory, 64 lanes x 64 columns at dtm) = A B for 64 x 64 x 64,
// A and B^T in the block layout at a_addr and b_addr (shared-memory
// addresses): eight K = 8 steps, the first one overwriting D.  One thread.
__device__ __forceinline__ void umma_64x64x64(uint32_t dtm, uint32_t a_addr, uint32_t b_addr)
{
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint64_t da = kmajor_desc(a_addr + 2 * k * CSB), db = kmajor_desc(b_addr + 2 * k * CSB);
        const uint32_t acc = k > 0;
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
                     ::"r"(dtm), "l"(da), "l"(db), "r"(kIdescTf32), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
    }
}

// The mbarrier at mbar receives one arrival when every tcgen05.mma this
// thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the mbarrier's phase of parity `parity` has completed, for at
// most limit_ns; false when it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_ns();
    for (;;) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}\n"
                     : "=r"(done)
                     : "r"(mbar), "r"(parity)
                     : "memory");
        if (done) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Generic-proxy writes to shared memory made visible to the tensor cores.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Rows 16 w .. 16 w + 15 (w = this warp) of the 64 x 64 fp32 matrix at
// tensor-memory column col of the allocation tm (M = 64 layout: row 16 w + i
// in lane 32 w + i), in the mma accumulator fragment layout:
// v[j][2 h + e] = D[16 w + g + 8 h][8 j + 2 q + e].  The whole warp.
__device__ __forceinline__ void tmem_rows16(uint32_t tm, int warp, uint32_t col, float (&v)[8][4])
{
    uint32_t r[32];
    const uint32_t a = tm + ((uint32_t)(32 * warp) << 16) + col;
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(a));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) (&v[0][0])[i] = __uint_as_float(r[i]);
}

// This warp's rows of a fragment-layout matrix written to the block layout at
// dst, rounded to tf32 (an A operand of the next products).
__device__ __forceinline__ void store_rows16_tf32(float* dst, const float (&v)[8][4], int r0, int g, int q)
{
    char* d8 = reinterpret_cast<char*>(dst);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8)
            *reinterpret_cast<float2*>(d8 + boff(r0 + g + 8 * h8, 8 * nt + 2 * q)) =
                make_float2(round_tf32(v[nt][2 * h8]), round_tf32(v[nt][2 * h8 + 1]));
}

// M^T rounded to tf32 into mt (block layout) from the slice ms (block
// layout): each thread transposes 4 x 4 tiles in registers, 16-byte loads
// and stores.  The whole CTA.
__device__ __forceinline__ void transpose_tf32(const float* ms, float* mt, int tid)
{
    const char* s8 = reinterpret_cast<const char*>(ms);
    char* d8 = reinterpret_cast<char*>(mt);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        // 256 tiles of 4 x 4 (rows 4 tr .., columns 4 tc ..); within 8 lanes
        // tr & 1 and tc & 1 both vary, so the loads and the stores each meet
        // at most 4 lanes on one 16-byte bank group
        const int t = tid + THREADS * i;
        const int tc = (t & 1) | (((t >> 3) & 7) << 1);
        const int tr = ((t >> 1) & 3) | ((t >> 6) << 2);
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = *reinterpret_cast<const float4*>(s8 + boff(4 * tr + k, 4 * tc));
        *reinterpret_cast<float4*>(d8 + boff(4 * tc + 0, 4 * tr)) =
            make_float4(round_tf32(v[0].x), round_tf32(v[1].x), round_tf32(v[2].x), round_tf32(v[3].x));
        *reinterpret_cast<float4*>(d8 + boff(4 * tc + 1, 4 * tr)) =
            make_float4(round_tf32(v[0].y), round_tf32(v[1].y), round_tf32(v[2].y), round_tf32(v[3].y));
        *reinterpret_cast<float4*>(d8 + boff(4 * tc + 2, 4 * tr)) =
            make_float4(round_tf32(v[0].z), round_tf32(v[1].z), round_tf32(v[2].z), round_tf32(v[3].z));
        *reinterpret_cast<float4*>(d8 + boff(4 * tc + 3, 4 * tr)) =
            make_float4(round_tf32(v[0].w), round_tf32(v[1].w), round_tf32(v[2].w), round_tf32(v[3].w));
    }
}

// Element (r, c) of a block-layout slice.
__device__ __forceinline__ float at(const float* ms, int r, int c)
{
    return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(ms) + boff(r, c));
}
__device__ __forceinline__ float2 at2(const float* ms, int r, int c)      // c even
{
    return *reinterpret_cast<const float2*>(reinterpret_cast<const char*>(ms) + boff(r, c));
}

// |det(I + alpha M)| (ok == true) by the register-blocked identity-split
// LU of the block-layout slice xs; ok == false when a pivot is below 1/2 in
// magnitude.  All threads call.  Thread (br, bc) updates its whole 4 x 8
// block at every step where the block reaches below and right of the pivot:
// entries in eliminated rows or columns are never read again, so they need
// no masking.
__device__ float absdet_near_identity(Smem& sm, const float* xs, float alpha, bool& ok)
{
    const int t = threadIdx.x, br = t >> 3, bc = t & 7;
    const char* x8 = reinterpret_cast<const char*>(xs);
    float e[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float4 v0 = *reinterpret_cast<const float4*>(x8 + boff(4 * br + r, 8 * bc));
        const float4 v1 = *reinterpret_cast<const float4*>(x8 + boff(4 * br + r, 8 * bc + 4));
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

// log|det(W)|, W = add_identity I + alpha M (M the block-layout slice xs),
// by LU with partial pivoting on a row-major copy in W (64 rows of ROWW
// words).  Returns NaN when a pivot column is zero.
__device__ double logdet_pivoted(Smem& sm, const float* xs, float* W, float alpha, int add_identity)
{
    const int t = threadIdx.x;
    for (int e = t; e < NN; e += THREADS) {
        const int i = e / N, j = e % N;
        float v = alpha * at(xs, i, j);
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

// Copies a token's slice into a slice buffer in the block layout (cp.async,
// committed as one group): per warp instruction 8 rows x 4 granules, so that
// each row's 64 contiguous bytes come in one piece and the 8 lanes that
// write one 128-byte core matrix hit distinct banks.
__device__ __forceinline__ void issue_slice(float* xs, const float* src)
{
    char* x8 = reinterpret_cast<char*>(xs);
#pragma unroll
    for (int i = 0; i < NN / 4 / THREADS; ++i) {
        const int gi = threadIdx.x + THREADS * i;               // 1024 granules of 16 bytes
        const int lane = gi & 31, blk = gi >> 5;                // 32 blocks of 8 rows x 4 granules
        const int row = 8 * (blk & 7) + (lane & 7), c4 = 4 * (blk >> 3) + (lane >> 3);
        cp_async16(x8 + boff(row, 4 * c4), src + row * N + 4 * c4);
    }
    asm volatile("cp.async.commit_group;\n" ::);
}


__global__ void __launch_bounds__(THREADS, 3)
k64_chunk_readout_tc(KParams p, const float* __restrict__ x, const float* __restrict__ u, int64_t snap_every,
                  float* __restrict__ o_out, float* __restrict__ snaps, float* __restrict__ totals,
                  uint32_t* status)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    float* ut = reinterpret_cast<float*>(smem_raw + sizeof(Smem));     // U transposed, [rq][N]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const int64_t chain = blockIdx.x;                // (b*H + h)*K + k, like the generic kernels
    const int64_t k = chain % p.K, bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    const int64_t tok = p.H * NN;
    const float* xb = x + (b * p.L * p.H + h) * NN;
    const int r0 = 16 * warp;                        // this warp's rows
    const bool detnorm = p.mode == MRU_MODE_DETNORM;
    const bool series = detnorm && p.add_identity != 0;
    constexpr uint64_t kWaitNs = 2000000000ull;      // bound of every tensor-core wait

    issue_slice(sm.mb[0], xb + t0 * tok);
    const int rq = p.rq;
    for (int e = tid; e < N * rq; e += THREADS) {
        const int j = e / rq, c = e - j * rq;
        ut[c * N + j] = u[h * p.u_hs + e];
    }
    for (int e = tid; e < NN; e += THREADS) sm.qa[e] = 0.0f;     // Q_{t0-1} = 0 (any layout)
    const uint32_t mbar = smem_u32(&sm.mbar);
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(smem_u32(&sm.tmem)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = sm.tmem;                     // columns 0-63: Q M; 64-127: M M, then M^2 M
    const uint32_t a_q = smem_u32(sm.qa), b_mt = smem_u32(sm.mt);
    uint32_t phase = 0;
    bool alive = true;

    float Qd[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) Qd[nt][i] = 0.0f;

    for (int64_t t = t0; t < t1 && alive; ++t) {
        const int cur = (int)((t - t0) & 1);
        const float* xs = sm.mb[cur];
        if (t + 1 < t1) issue_slice(sm.mb[cur ^ 1], xb + (t + 1) * tok);
        else asm volatile("cp.async.commit_group;\n" ::);
        asm volatile("cp.async.wait_group 1;\n" ::);
        __syncthreads();
        transpose_tf32(xs, sm.mt, tid);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            umma_64x64x64(tm, a_q, b_mt);                              // Q_{t-1} M
            if (series) umma_64x64x64(tm + 64, smem_u32(xs), b_mt);    // M M
            umma_commit(mbar);
        }
        alive = __syncthreads_and(mbar_wait(mbar, phase, kWaitNs));
        phase ^= 1;
        if (!alive) break;
        tc_fence_after();

        // ---- determinant scale ----
        float ca = p.alpha, dv = p.add_identity ? 0.0f : -1.0f;
        if (detnorm) {
            bool ok = false;
            float cm1 = 0.0f;
            if (series) {
                // log det(I + E), E = alpha M, by its trace series
                //   tr E - tr E^2 / 2 + tr E^3 / 3 - tr E^4 / 4 + R,
                // tr E^k = <E^(k-1), E^T> from M2 = M M and M3 = M2 M (tf32
                // products on the tensor cores).  Since tr E^k = <E^(k-3), (E^3)^T>
                // and |E^m|_F <= |E^2|_F |E|_F^(m-2),
                //   |R| <= |E^3|_F |E^2|_F / (5 (1 - |E|_F))   (|E|_F < 1),
                // the series is taken when that bound is at most 1e-6 (the scale
                // c = exp(-log det / 64) then good to 1.6e-8; the tf32 rounding of
                // the products' operands adds well under 1e-7 to log det at the
                // workload's alpha).
                float M2[8][4];
                tmem_rows16(tm, warp, 64, M2);
                float tr1 = 0.0f, tr2 = 0.0f, tr3 = 0.0f, tr4 = 0.0f, n1 = 0.0f, n2 = 0.0f, n3 = 0.0f;
                if (lane < 16) tr1 = at(xs, r0 + lane, r0 + lane);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                        const float2 mv = at2(xs, row, col);
                        const float mt0 = at(xs, col, row), mt1 = at(xs, col + 1, row);   // M^T here
                        tr2 = fmaf(mv.x, mt0, fmaf(mv.y, mt1, tr2));
                        tr3 = fmaf(M2[nt][2 * h8], mt0, fmaf(M2[nt][2 * h8 + 1], mt1, tr3));
                        n1 = fmaf(mv.x, mv.x, fmaf(mv.y, mv.y, n1));
                        n2 = fmaf(M2[nt][2 * h8], M2[nt][2 * h8], fmaf(M2[nt][2 * h8 + 1], M2[nt][2 * h8 + 1], n2));
                    }
                // M3 = M2 M: M2 goes where Q_{t-1} was (its product is done)
                store_rows16_tf32(sm.qa, M2, r0, g, q);
                fence_async_smem();
                tc_fence_before();
                __syncthreads();
                tc_fence_after();
                if (tid == 0) {
                    umma_64x64x64(tm + 64, a_q, b_mt);
                    umma_commit(mbar);
                }
                alive = __syncthreads_and(mbar_wait(mbar, phase, kWaitNs));
                phase ^= 1;
                if (!alive) break;
                tc_fence_after();
                {
                    float M3[8][4];
                    tmem_rows16(tm, warp, 64, M3);
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                        for (int h8 = 0; h8 < 2; ++h8) {
                            const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                            const float mt0 = at(xs, col, row), mt1 = at(xs, col + 1, row);
                            tr4 = fmaf(M3[nt][2 * h8], mt0, fmaf(M3[nt][2 * h8 + 1], mt1, tr4));
                            n3 = fmaf(M3[nt][2 * h8], M3[nt][2 * h8], fmaf(M3[nt][2 * h8 + 1], M3[nt][2 * h8 + 1], n3));
                        }
                }
                tr1 = warp_sum(tr1);
                tr2 = warp_sum(tr2);
                tr3 = warp_sum(tr3);
                tr4 = warp_sum(tr4);
                n1 = warp_sum(n1);
                n2 = warp_sum(n2);
                n3 = warp_sum(n3);
                if (lane == 0) {
                    float* rd = sm.red[warp];
                    rd[0] = tr1; rd[1] = tr2; rd[2] = tr3; rd[3] = tr4; rd[4] = n1; rd[5] = n2; rd[6] = n3;
                }
                __syncthreads();
                float v[7];
#pragma unroll
                for (int i = 0; i < 7; ++i) v[i] = (sm.red[0][i] + sm.red[1][i]) + (sm.red[2][i] + sm.red[3][i]);
                const float a = p.alpha, a2 = a * a;
                const float ld = a * v[0] - a2 * (0.5f * v[1]) + a2 * a * (v[2] * (1.0f / 3.0f)) -
                                 a2 * a2 * (0.25f * v[3]);
                const float fe = a * sqrtf(v[4]), fe2 = a2 * sqrtf(v[5]), fe3 = a2 * a * sqrtf(v[6]);
                const float bound = fe3 * fe2 / (5.0f * (1.0f - fe));
                ok = fe < 1.0f && bound <= 1e-6f;      // false for non-finite inputs too
                if (ok) cm1 = expm1f(-ld * (1.0f / N));
            }
            if (!ok) {
                // near the identity: |det| = prod (1 + delta_k) in fp32 (64
                // factors near 1, relative error about 2e-7), c - 1 =
                // expm1(-log1p(|det| - 1) / 64); otherwise the pivoted LU's fp64
                // sum, on a row-major copy in mt and qa (no product reads them now)
                bool near = p.add_identity != 0;
                if (near) cm1 = expm1f(-log1pf(absdet_near_identity(sm, xs, p.alpha, near) - 1.0f) * (1.0f / N));
                __syncthreads();
                const bool retry = __syncthreads_or(!near);
                bool bad = false;
                if (retry) {
                    const double ld = logdet_pivoted(sm, xs, sm.mt, p.alpha, p.add_identity);
                    bad = !isfinite(ld);
                    cm1 = (float)expm1(-ld / N);
                }
                ok = !bad;
            }
            const float c = 1.0f + cm1;
            if (!ok || !isfinite(cm1) || !(c > 0.0f)) {
                if (tid == 0) atomicOr(status, STATUS_SINGULAR);
                ca = 0.0f;
                dv = 0.0f;
            } else {
                ca = c * p.alpha;
                dv = p.add_identity ? cm1 : -1.0f;
            }
        }
        // ---- Q_t = Q + (F + Q F), Q F = ca Q M + dv Q, F = ca M + dv I ----
        {
            float P[8][4];
            tmem_rows16(tm, warp, 0, P);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                    const float2 xv = at2(xs, row, col);
                    float f0 = ca * xv.x, f1 = ca * xv.y;
                    if (row == col) f0 += dv;
                    if (row == col + 1) f1 += dv;
                    const float q0 = fmaf(ca, P[nt][2 * h8], dv * Qd[nt][2 * h8]);
                    const float q1 = fmaf(ca, P[nt][2 * h8 + 1], dv * Qd[nt][2 * h8 + 1]);
                    Qd[nt][2 * h8] += f0 + q0;
                    Qd[nt][2 * h8 + 1] += f1 + q1;
                }
        }
        // ---- readout of the local prefix: V_t = Q_t U (rq columns; the loop
        // bound is uniform over the CTA, so every lane reaches the shuffles) ----
        const int64_t row_bth = (b * p.L + t) * p.H + h;
        for (int c = 0; c < rq; ++c) {
            float ur[8][2];                          // U[:, c] at this lane's columns 8 nt + 2 q, + 1
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const float2 v = *reinterpret_cast<const float2*>(ut + c * N + 8 * nt + 2 * q);
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
        // Q_t, rounded, is the next token's A operand; the slice buffer and mt
        // are reused after the barrier
        store_rows16_tf32(sm.qa, Qd, r0, g, q);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (!alive) {
        if (tid == 0) atomicOr(status, STATUS_TIMEOUT);
    } else {
        float* tot = totals + chain * NN;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8)
                *reinterpret_cast<float2*>(tot + (r0 + g + 8 * h8) * N + 8 * nt + 2 * q) =
                    make_float2(Qd[nt][2 * h8], Qd[nt][2 * h8 + 1]);
    }
    asm volatile("cp.async.wait_all;\n" ::);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tm));
}

}  // namespace tc

}  // namespace

// The chunk phase on tcgen05 instead of mma.sync (read at every call).
bool use_tcgen05()
{
    const char* v = getenv("MRU_N64_TCGEN05");
    return v != nullptr && v[0] == '1' && v[1] == 0;
}

// The readout form (tf32 unless another arithmetic is asked for), and every
// state when tf32 is asked for explicitly: the chunk kernel then records each
// Q_t as a snapshot and the fix-up writes S_t = C + C Q_t for every token.
bool supports(const KParams& p, bool readout)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_F32 && p.K > 1 &&
           (p.mode == MRU_MODE_DETNORM || p.mode == MRU_MODE_RESHAPE) &&
           (readout ? (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_TF32) : p.math == MRU_MATH_TF32);
}

cudaError_t launch_chunk_readout(const KParams& p, const float* x, const float* u, int64_t snap_every,
                                 float* o_out, float* snaps, float* totals, uint32_t* status, cudaStream_t s)
{
    const int64_t chains = p.B * p.H * p.K;
    if (use_tcgen05()) {
        const size_t sm = sizeof(tc::Smem) + sizeof(float) * N * p.rq;
        cudaError_t e = cudaFuncSetAttribute(tc::k64_chunk_readout_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)sm);
        if (e != cudaSuccess) return e;
        tc::k64_chunk_readout_tc<<<(unsigned)chains, THREADS, sm, s>>>(p, x, u, snap_every, o_out, snaps, totals,
                                                                        status);
        return cudaGetLastError();
    }
    const size_t sm = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(k64_chunk_readout, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k64_chunk_readout<<<(unsigned)chains, THREADS, sm, s>>>(p, x, u, snap_every, o_out, snaps, totals, status);
    return cudaGetLastError();
}

cudaError_t launch_fixup_readout(const KParams& p, const float* carry, const float* u, int64_t snap_every,
                                 float* o_out, float* snaps, cudaStream_t s)
{
    const int64_t chains = p.B * p.H * p.K;
    if (chains == 0) return cudaSuccess;
    const size_t sm = sizeof(float) * (2 * FX_BUF + N * p.rq);
    cudaError_t e = cudaFuncSetAttribute(k64_fixup, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k64_fixup<<<(unsigned)chains, THREADS, sm, s>>>(p, carry, u, snap_every, o_out, snaps);
    return cudaGetLastError();
}

}  // namespace n64
}  // namespace mru
