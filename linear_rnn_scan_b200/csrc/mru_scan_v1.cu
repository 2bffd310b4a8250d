// mru_scan_v1.cu -- generic (every supported n) chunked prefix-product scan.
//
// The scan follows the method's associativity argument ("MRU Update: An
// independent developer's alternative to Attention is now running
// successfully", section "What MRU Actually Does"): the sequence of each
// (b, h) is cut into chunks of C tokens; every chunk forms its local prefix
// products independently, the chunk totals are scanned, and every local
// prefix is then multiplied on the left by its chunk's carry.
//
// Numerics.  Every matrix is carried in identity-split form, X = I + F,
// P = I + Q, so that the near-identity inputs of the determinant-corrected
// workloads lose nothing to the implicit 1 on the diagonal:
//     Q_t = Q_{t-1} + (F_t + Q_{t-1} F_t)          (in-chunk, fp32)
//     carry_{k+1} = carry_k + carry_k Q_k          (chunk totals, fp64)
//     S_t = carry + carry Q_t                      (fix-up, fp32)
// The chunk-total scan is two-level (groups of G totals, then the group
// totals) so that no serial chain is longer than max(G, K/G).
//
// Kernels (one call of mru_scan_fused):
//   k_chunk_prefix  one CTA per (b, h, chunk): lift + in-chunk prefix; writes
//                   Q_t where S_t (or o_t = S_t u, snapshots) will go, and
//                   the chunk total to the workspace
//   k_carry_local   one CTA per (b, h, group): in-group inclusive prefixes
//   k_carry_groups  one CTA per (b, h): exclusive group carries (serial)
//   k_carry_final   one CTA per (b, h, chunk): exclusive chunk carries
//   k_fixup         one CTA per (b, h, chunk): S_t = carry (I + Q_t) in place
#include <type_traits>

#include "mru_internal.cuh"

namespace mru {
namespace {

constexpr int kThreads = 256;

// Thread groups that run the per-token routines below: a whole CTA of
// kThreads threads (barriers are __syncthreads), or one warp that owns a
// chain by itself (barriers are __syncwarp; used for n <= 16, where a warp
// covers a matrix in eight elements per lane and no CTA-wide barrier is
// worth its latency).
struct CtaGroup {
    static constexpr int kSize = kThreads;
    __device__ static int idx() { return threadIdx.x; }
    __device__ static void sync() { __syncthreads(); }
};
struct WarpGroup {
    static constexpr int kSize = 32;
    __device__ static int idx() { return threadIdx.x & 31; }
    __device__ static void sync() { __syncwarp(); }
};

__device__ __forceinline__ float load_elem(const void* base, int64_t idx, int dtype)
{
    if (dtype == MRU_BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
    return reinterpret_cast<const float*>(base)[idx];
}

// Trailing-submatrix update of one elimination step on an N x N matrix in
// shared memory: W[i][j] -= W[i][k] * r * W[k][j] for i, j > k.
template <int N, class Grp = CtaGroup>
__device__ __forceinline__ void eliminate_step(float* sW, int k, float r)
{
    const int m = N - k - 1;
    for (int idx = Grp::idx(); idx < m * m; idx += Grp::kSize) {
        const int i = k + 1 + idx / m, j = k + 1 + idx % m;
        sW[i * N + j] = fmaf(-sW[i * N + k] * r, sW[k * N + j], sW[i * N + j]);
    }
}

// Per-token scalars in shared memory, after the 4N floats of per-row
// scratch: [4N] pivot row (int), [4N+1] flag, [4N+2..4N+3] log|det| (fp64),
// [4N+4] c, [4N+5] c - 1.  (The scratch area holds 4N + 8 floats.)
template <int N> __device__ __forceinline__ int* aux_piv(float* a) { return reinterpret_cast<int*>(a + 4 * N); }
template <int N> __device__ __forceinline__ float* aux_flag(float* a) { return a + 4 * N + 1; }
template <int N> __device__ __forceinline__ double* aux_logdet(float* a) { return reinterpret_cast<double*>(a + 4 * N + 2); }
template <int N> __device__ __forceinline__ float* aux_c(float* a) { return a + 4 * N + 4; }

// log|det W| by LU with partial pivoting on the full matrix in sW (destroyed),
// accumulated in fp64 into the logdet slot; the flag slot is set when a pivot
// column is entirely zero.  Called by the whole CTA.
template <int N, class Grp = CtaGroup>
__device__ void cta_logabsdet_pivoted(float* sW, float* sAux)
{
    int* sPiv = aux_piv<N>(sAux);
    if (Grp::idx() == 0) { *aux_logdet<N>(sAux) = 0.0; *aux_flag<N>(sAux) = 0.0f; }
    Grp::sync();
    for (int k = 0; k < N; ++k) {
        if (Grp::idx() < 32) {
            float best = -1.0f;
            int bi = k;
            for (int i = k + Grp::idx(); i < N; i += 32) {
                const float a = fabsf(sW[i * N + k]);
                if (a > best) { best = a; bi = i; }
            }
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_down_sync(0xffffffffu, best, o);
                const int oi = __shfl_down_sync(0xffffffffu, bi, o);
                if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            if (Grp::idx() == 0) {
                *sPiv = bi;
                if (!(best > 0.0f)) *aux_flag<N>(sAux) = 1.0f;
            }
        }
        Grp::sync();
        const int piv = *sPiv;
        if (piv != k) {
            for (int j = Grp::idx(); j < N; j += Grp::kSize) {
                const float a = sW[k * N + j];
                sW[k * N + j] = sW[piv * N + j];
                sW[piv * N + j] = a;
            }
        }
        Grp::sync();
        const float pk = sW[k * N + k];
        if (Grp::idx() == 0) *aux_logdet<N>(sAux) += log(fabs((double)pk));
        const float r = (pk != 0.0f) ? 1.0f / pk : 0.0f;
        eliminate_step<N, Grp>(sW, k, r);
        Grp::sync();
    }
}

// D = (A + A Y) * scale = A (I + Y) * scale for N x N matrices in shared
// memory (D distinct from A and Y); ends with a barrier.  The product term
// is accumulated on its own before A is added.
template <int N, class Grp = CtaGroup>
__device__ __forceinline__ void cta_mul_plus(const float* A, const float* Y, float* D, float scale)
{
    for (int e = Grp::idx(); e < N * N; e += Grp::kSize) {
        const int i = e / N, j = e % N;
        float a = 0.0f;
#pragma unroll 8
        for (int q = 0; q < N; ++q) a = fmaf(A[i * N + q], Y[q * N + j], a);
        D[e] = (A[e] + a) * scale;
    }
    Grp::sync();
}

// Scaling and Taylor degree of exp(A) for the N x N matrix A in shared
// memory: the least s >= 0 with ||A||_1 / 2^s <= 1/2, and the least degree m
// (1 <= m <= 12) whose next Taylor term ||B||^(m+1) / (m+1)! of B = A / 2^s
// is below 2^-26 ||B||.  The whole CTA calls it; the results are uniform.
template <int N, class Grp = CtaGroup>
__device__ void expm_plan(const float* A, float* sAux, int& m, int& sq)
{
    for (int j = Grp::idx(); j < N; j += Grp::kSize) {
        float c = 0.0f;
        for (int i = 0; i < N; ++i) c += fabsf(A[i * N + j]);
        sAux[j] = c;
    }
    Grp::sync();
    int* cfg = reinterpret_cast<int*>(sAux + 4 * N);
    if (Grp::idx() == 0) {
        float nrm = 0.0f;
        for (int j = 0; j < N; ++j) nrm = fmaxf(nrm, sAux[j]);
        int s2 = 0;
        while (nrm > 0.5f && s2 < 64) { nrm *= 0.5f; ++s2; }     // nrm = ||B||_1 <= 1/2 (finite input)
        int d = 1;
        float term = nrm;                     // ||B||^d / d!
        while (d < 12 && term * nrm / (float)(d + 1) > 1.4901161e-8f * nrm) {
            term = term * nrm / (float)(d + 1);
            ++d;
        }
        cfg[0] = d;
        cfg[1] = s2;
    }
    Grp::sync();
    m = cfg[0];
    sq = cfg[1];
    Grp::sync();
}

// Orthogonal constructions of the skew-symmetric part A = alpha (M - M^T) / 2
// of the slice M (in sM), written as F = X - I into sF:
//   Cayley map   X = (I - A)^-1 (I + A), so F = 2 (I - A)^-1 A: Gauss-Jordan
//                elimination of I - A (kept as I + E, E = -A) applied to 2A.
//                The symmetric part of I - A is I, so every pivot is at
//                least 1 and no pivoting is needed;
//   exponential  X = exp(A) by scaling and squaring: B = A / 2^s with
//                ||B||_1 <= 1/2, exp(B) - I from its Taylor polynomial of
//                degree m (Horner, Y_m = B / m, Y_k = B (I + Y_{k+1}) / k,
//                F = Y_1; m is the least degree whose next term
//                ||B||^(m+1) / (m+1)! is below 2^-26 ||B||), then s
//                squarings (I + F)^2 - I = 2F + F F.
// sW and sAux are scratch, and so is sM in the exponential mode (the slice is
// not kept); the whole CTA calls it; ends with a barrier.
template <int N, class Grp = CtaGroup>
__device__ void cta_orthogonal(const KParams& p, float* sF, float* sM, float* sW, float* sAux)
{
    constexpr int NN = N * N;
    const int tid = Grp::idx();
    const float ha = 0.5f * p.alpha;
    if (p.mode == MRU_MODE_CAYLEY) {
        for (int e = tid; e < NN; e += Grp::kSize) {
            const int i = e / N, j = e % N;
            const float a = ha * (sM[e] - sM[j * N + i]);
            sW[e] = -a;                       // I - A = I + E
            sF[e] = 2.0f * a;                 // right-hand side 2A
        }
        Grp::sync();
        for (int k = 0; k < N; ++k) {
            const float r = 1.0f / (1.0f + sW[k * N + k]);
            for (int i = tid; i < N; i += Grp::kSize) sAux[i] = sW[i * N + k] * r;
            Grp::sync();
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                if (i == k) continue;             // the pivot row stays as it is
                const float f = sAux[i];
                sF[e] = fmaf(-f, sF[k * N + j], sF[e]);
                if (j > k) sW[e] = fmaf(-f, sW[k * N + j], sW[e]);
            }
            Grp::sync();
        }
        for (int e = tid; e < NN; e += Grp::kSize) {
            const int i = e / N;
            sF[e] = sF[e] / (1.0f + sW[i * N + i]);
        }
        Grp::sync();
        return;
    }
    // exponential
    for (int e = tid; e < NN; e += Grp::kSize) {
        const int i = e / N, j = e % N;
        sW[e] = ha * (sM[e] - sM[j * N + i]);
    }
    Grp::sync();
    int m, sq;
    expm_plan<N, Grp>(sW, sAux, m, sq);
    const float scale = ldexpf(1.0f, -sq);
    for (int e = tid; e < NN; e += Grp::kSize) sW[e] *= scale;             // B
    Grp::sync();
    float* cur = sF;
    float* nxt = sM;                                                     // M is no longer needed
    for (int e = tid; e < NN; e += Grp::kSize) cur[e] = sW[e] * (1.0f / (float)m);
    Grp::sync();
    for (int k = m - 1; k >= 1; --k) {
        cta_mul_plus<N, Grp>(sW, cur, nxt, 1.0f / (float)k);
        float* t = cur; cur = nxt; nxt = t;
    }
    for (int r = 0; r < sq; ++r) {
        for (int e = tid; e < NN; e += Grp::kSize) {
            const int i = e / N, j = e % N;
            float a = 0.0f;
#pragma unroll 8
            for (int q = 0; q < N; ++q) a = fmaf(cur[i * N + q], cur[q * N + j], a);
            nxt[e] = 2.0f * cur[e] + a;
        }
        Grp::sync();
        float* t = cur; cur = nxt; nxt = t;
    }
    if (cur != sF) {
        for (int e = tid; e < NN; e += Grp::kSize) sF[e] = cur[e];
        Grp::sync();
    }
}

// Lift one token-head slice into F = X - I (shared memory, sF).  The whole
// CTA calls it; it ends with a barrier.  sM, sW: N*N floats of scratch;
// sAux: 4N + 8 floats of scratch.
//
// The per-token scalars that every later step multiplies into the product
// (the determinant scale c and c - 1, the LDU diagonal D_i - 1) are formed in
// fp64 and rounded once: a bias of one fp32 ulp in them would otherwise add
// up coherently over thousands of tokens.
template <int N, class Grp = CtaGroup>
__device__ void cta_construct(const KParams& p, const void* src, int64_t off, float* sF,
                              float* sM, float* sW, float* sAux, uint32_t* status)
{
    constexpr int NN = N * N;
    const int tid = Grp::idx();
    if (p.src != SRC_EMBEDDING) {
        const float* f = reinterpret_cast<const float*>(src) + off;
        for (int e = tid; e < NN; e += Grp::kSize) {
            float v = f[e];
            if (p.src == SRC_X && (e / N) == (e % N)) v -= 1.0f;
            sF[e] = v;
        }
        Grp::sync();
        return;
    }
    for (int e = tid; e < NN; e += Grp::kSize) sM[e] = load_elem(src, off + e, p.x_dtype);
    Grp::sync();

    if (p.mode == MRU_MODE_RESHAPE) {
        for (int e = tid; e < NN; e += Grp::kSize) {
            float v = p.alpha * sM[e];
            if (!p.add_identity && (e / N) == (e % N)) v -= 1.0f;
            sF[e] = v;
        }
        Grp::sync();
        return;
    }

    if (p.mode == MRU_MODE_CAYLEY || p.mode == MRU_MODE_EXPM) {
        cta_orthogonal<N, Grp>(p, sF, sM, sW, sAux);
        return;
    }

    if (p.mode == MRU_MODE_LDU) {
        // D_k and D_k - 1 (the latter without cancellation), fp64 then rounded.
        for (int k = tid; k < N; k += Grp::kSize) {
            const double z = (double)p.ldu_d * tanh((double)sM[k * N + k]);
            sAux[k] = (float)exp(z);
            sAux[N + k] = (float)expm1(z);
        }
        Grp::sync();
        const float a = p.ldu_a;
        // X_ij = sum_{k <= min(i,j)} L_ik D_k U_kj with unit diagonals.
        for (int e = tid; e < NN; e += Grp::kSize) {
            const int i = e / N, j = e % N;
            const int m = i < j ? i : j;
            float acc = 0.0f;
            for (int k = 0; k < m; ++k)
                acc = fmaf(a * sM[i * N + k] * sAux[k], a * sM[k * N + j], acc);
            if (i < j) acc = fmaf(sAux[i], a * sM[i * N + j], acc);
            else if (i > j) acc = fmaf(a * sM[i * N + j], sAux[j], acc);
            else acc += sAux[N + i];
            sF[e] = acc;
        }
        Grp::sync();
        return;
    }

    // DETNORM: X = Xr * c, c = |det Xr|^(-1/N).
    bool need_pivot = !p.add_identity;
    if (p.add_identity) {
        // Near-identity fast path: eliminate W = I + E keeping only E, so the
        // pivots 1 + delta_k are known through delta_k to full precision;
        // |det| = prod |1 + delta_k| is formed in fp64.  Falls back to
        // pivoting when a pivot is small.
        for (int e = tid; e < NN; e += Grp::kSize) sW[e] = p.alpha * sM[e];
        Grp::sync();
        for (int k = 0; k < N; ++k) {
            const float r = 1.0f / (1.0f + sW[k * N + k]);
            eliminate_step<N, Grp>(sW, k, r);
            Grp::sync();
        }
        if (tid == 0) {
            double prod = 1.0;
            float bad = 0.0f;
            for (int k = 0; k < N; ++k) {
                const float d = sW[k * N + k];
                if (!(fabsf(1.0f + d) >= 0.5f)) bad = 1.0f;
                prod *= 1.0 + (double)d;
            }
            *aux_logdet<N>(sAux) = log(fabs(prod));
            *aux_flag<N>(sAux) = bad;
        }
        Grp::sync();
        need_pivot = *aux_flag<N>(sAux) != 0.0f;
        Grp::sync();
    }
    if (need_pivot) {
        for (int e = tid; e < NN; e += Grp::kSize) {
            float v = p.alpha * sM[e];
            if (p.add_identity && (e / N) == (e % N)) v += 1.0f;
            sW[e] = v;
        }
        Grp::sync();
        cta_logabsdet_pivoted<N, Grp>(sW, sAux);
    }
    if (tid == 0) {
        const double ld = *aux_logdet<N>(sAux);
        const bool singular = need_pivot && *aux_flag<N>(sAux) != 0.0f;
        const double cm1 = expm1(-ld / N);
        float c = (float)(1.0 + cm1);
        float cm1f = (float)cm1;
        if (singular || !isfinite(ld) || !isfinite(c) || c == 0.0f) {
            atomicOr(status, STATUS_SINGULAR);
            c = 0.0f;        // output unspecified; keep it finite (X = I)
            cm1f = 0.0f;
        }
        aux_c<N>(sAux)[0] = c;
        aux_c<N>(sAux)[1] = cm1f;
    }
    Grp::sync();
    const float c = aux_c<N>(sAux)[0];
    const float cm1 = aux_c<N>(sAux)[1];
    for (int e = tid; e < NN; e += Grp::kSize) {
        const bool diag = (e / N) == (e % N);
        float v = c * (p.alpha * sM[e]);
        if (diag) v += p.add_identity ? cm1 : -1.0f;
        if (c == 0.0f) v = 0.0f;
        sF[e] = v;
    }
    Grp::sync();
}

// ----------------------------------------------------------------------------
template <int N>
__global__ void __launch_bounds__(kThreads)
k_build_states(KParams p, const void* src, float* X_out, int store_minus_identity, uint32_t* status)
{
    constexpr int NN = N * N;
    extern __shared__ float smem[];
    float* sF = smem;
    float* sM = sF + NN;
    float* sW = sM + NN;
    float* sAux = sW + NN;
    const int64_t rows = p.B * p.L * p.H;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        cta_construct<N>(p, src, row * NN, sF, sM, sW, sAux, status);
        for (int e = threadIdx.x; e < NN; e += kThreads) {
            float v = sF[e];
            if (!store_minus_identity && (e / N) == (e % N)) v += 1.0f;
            X_out[row * NN + e] = v;
        }
        __syncthreads();
    }
}

template <int N, class Grp>
__global__ void __launch_bounds__(kThreads)
k_chunk_prefix(KParams p, const void* src, const float* u, int64_t snap_every, float* S_out,
               float* o_out, float* snaps, float* totals, uint32_t* status, const float* S0, int direct, int gfl)
{
    constexpr int NN = N * N;
    constexpr int PER = (NN + Grp::kSize - 1) / Grp::kSize;
    extern __shared__ float smem[];
    constexpr int GPB = kThreads / Grp::kSize;     // chains per CTA (one per group)
    const int gi = threadIdx.x / Grp::kSize;
    const int64_t chain = (int64_t)blockIdx.x * GPB + gi;
    if (chain >= p.B * p.H * p.K) return;          // the whole group leaves together
    float* sQ = smem + (size_t)gi * gfl;
    float* sF = sQ + NN;
    float* sM = sF + NN;
    float* sW = sM + NN;
    float* sAux = sW + NN;
    float* sU = sAux + 4 * N + 8;
    const int tid = Grp::idx();
    const int64_t k = chain % p.K;
    const int64_t bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    const bool readout = o_out != nullptr;

    const int rq = p.rq;                    // readout query columns
    // direct (one chunk per sequence): the chain starts from S0 (or I), and
    // every output is final; otherwise from I, fixed up later
    for (int e = tid; e < NN; e += Grp::kSize)
        sQ[e] = (direct && S0) ? S0[bh * NN + e] - ((e / N == e % N) ? 1.0f : 0.0f) : 0.0f;
    const float one = direct ? 1.0f : 0.0f;
    if (readout)
        for (int e = tid; e < N * rq; e += Grp::kSize) sU[e] = u[h * p.u_hs + e];
    Grp::sync();

    for (int64_t t = t0; t < t1; ++t) {
        const int64_t row = (b * p.L + t) * p.H + h;
        cta_construct<N, Grp>(p, src, row * NN, sF, sM, sW, sAux, status);
        float acc[PER];
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int e = tid + r * Grp::kSize;
            if (e < NN) {
                const int i = e / N, j = e % N;
                // The product term is accumulated on its own (its magnitude is
                // that of F) and only then added to Q: accumulating on top of
                // Q + F would round every partial sum at the scale of Q.
                float a = 0.0f;
#pragma unroll 8
                for (int q = 0; q < N; ++q) a = fmaf(sQ[i * N + q], sF[q * N + j], a);
                acc[r] = sQ[e] + (sF[e] + a);
            }
        }
        Grp::sync();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int e = tid + r * Grp::kSize;
            if (e < NN) {
                sQ[e] = acc[r];
                if (!readout) S_out[row * NN + e] = acc[r] + ((e / N == e % N) ? one : 0.0f);
            }
        }
        Grp::sync();
        if (readout) {
            for (int e = tid; e < N * rq; e += Grp::kSize) {
                const int i = e / rq, c = e - i * rq;
                float v = 0.0f;
                for (int j = 0; j < N; ++j) v = fmaf(sQ[i * N + j], sU[j * rq + c], v);
                o_out[row * N * rq + e] = v + one * sU[i * rq + c];   // Q_t U (+ U when final)
            }
            if (snap_every > 0 && ((t + 1) % snap_every) == 0) {
                const int64_t srow = (b * (p.L / snap_every) + (t + 1) / snap_every - 1) * p.H + h;
                for (int e = tid; e < NN; e += Grp::kSize)
                    snaps[srow * NN + e] = sQ[e] + ((e / N == e % N) ? one : 0.0f);
            }
        }
    }
    if (!direct)
        for (int e = tid; e < NN; e += Grp::kSize) totals[chain * NN + e] = sQ[e];
}

// fp64 products of the chunk-total scan.  n >= 32: the CTA's 8 warps on the
// fp64 tensor cores (mma.sync m8n8k4) from shared-memory tiles with rows
// padded to n + 4 doubles (the fragment reads of a half-warp then hit 16
// distinct 8-byte banks); warp w computes rows 8 MT (w / 2) ... and columns
// 8 NT (w % 2) ..., MT x NT tiles of 8 x 8.  n < 32: one output element per
// thread on the SIMT fp64 pipe.
template <int N>
struct CarryMul {
    static constexpr bool kTensor = N >= 32;
    static constexpr int SP = kTensor ? N + 4 : N;            // shared-memory row stride
    static constexpr int PER = (N * N + kThreads - 1) / kThreads;
    static constexpr int MT = kTensor ? N / 32 : 1, NT = kTensor ? N / 16 : 1;   // tiles per warp (tensor path)

    __device__ static void pos(int r, int& row, int& col)
    {
        if constexpr (kTensor) {
            const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
            const int tile = r >> 1, mt = tile / NT, nt = tile % NT;
            row = 8 * MT * (w >> 1) + 8 * mt + (lane >> 2);
            col = 8 * NT * (w & 1) + 8 * nt + 2 * (lane & 3) + (r & 1);
        } else {
            const int e = threadIdx.x + r * kThreads;
            row = e / N;
            col = e % N;
        }
    }
    __device__ static bool valid(int r) { return kTensor || threadIdx.x + r * kThreads < N * N; }

    // acc[r] = (A B)[pos(r)], A and B N x N fp64 in shared memory (stride SP).
    __device__ static void mul(const double* A, const double* Bm, double (&acc)[PER])
    {
        if constexpr (kTensor) {
            const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
            const int r0 = 8 * MT * (w >> 1), c0 = 8 * NT * (w & 1);
            double d[2][MT][NT][2];
#pragma unroll
            for (int i = 0; i < 2 * MT * NT * 2; ++i) (&d[0][0][0][0])[i] = 0.0;
#pragma unroll 4
            for (int kk = 0; kk < N / 4; ++kk) {
                double av[MT], bv[NT];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) av[mt] = A[(r0 + 8 * mt + g) * SP + 4 * kk + t];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) bv[nt] = Bm[(4 * kk + t) * SP + c0 + 8 * nt + g];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        double (&dd)[2] = d[kk & 1][mt][nt];
                        asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
                                     : "+d"(dd[0]), "+d"(dd[1])
                                     : "d"(av[mt]), "d"(bv[nt]));
                    }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) acc[2 * (mt * NT + nt) + h] = d[0][mt][nt][h] + d[1][mt][nt][h];
        } else {
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                const int e = threadIdx.x + r * kThreads;
                double a = 0.0;
                if (e < N * N) {
                    const int i = e / N, c = e % N;
                    for (int q = 0; q < N; ++q) a = fma(A[i * SP + q], Bm[q * SP + c], a);
                }
                acc[r] = a;
            }
        }
    }
};
static_assert(CarryMul<64>::PER == 2 * CarryMul<64>::MT * CarryMul<64>::NT, "tile outputs per thread");
static_assert(CarryMul<32>::PER == 2 * CarryMul<32>::MT * CarryMul<32>::NT, "tile outputs per thread");
static_assert(CarryMul<16>::MT * CarryMul<16>::NT == 1 && CarryMul<8>::MT * CarryMul<8>::NT == 1 &&
                  CarryMul<4>::MT * CarryMul<4>::NT == 1,
              "the SIMT path keeps one tile");

// In-group inclusive prefixes of the chunk totals, fp64, split form:
// R_j = R_{j-1} + T_j + R_{j-1} T_j.
template <int N>
__global__ void __launch_bounds__(kThreads)
k_carry_local(KParams p, const float* totals, double* local)
{
    constexpr int NN = N * N;
    using CM = CarryMul<N>;
    constexpr int SP = CM::SP, PER = CM::PER;
    extern __shared__ double dsm[];
    double* sR = dsm;
    double* sT = sR + N * SP;
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x / p.NG, g = blockIdx.x % p.NG;
    const int64_t j0 = g * p.group;
    const int64_t j1 = (j0 + p.group < p.K) ? j0 + p.group : p.K;
    for (int e = tid; e < N * SP; e += kThreads) sR[e] = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
        const int64_t base = (bh * p.K + j) * NN;
        for (int e = tid; e < NN; e += kThreads) sT[(e / N) * SP + e % N] = (double)totals[base + e];
        __syncthreads();
        double acc[PER];
        CM::mul(sR, sT, acc);
        __syncthreads();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            if (!CM::valid(r)) continue;
            int row, col;
            CM::pos(r, row, col);
            const double v = sR[row * SP + col] + (sT[row * SP + col] + acc[r]);
            sR[row * SP + col] = v;
            local[base + row * N + col] = v;
        }
    }
}

// Exclusive group carries (full matrices, fp64): GC_0 = S0 (or I),
// GC_{g+1} = GC_g + GC_g R_{g,last}.  Serial over the groups of a sequence.
template <int N>
__global__ void __launch_bounds__(kThreads)
k_carry_groups(KParams p, const float* S0, const double* local, double* gcarry)
{
    constexpr int NN = N * N;
    using CM = CarryMul<N>;
    constexpr int SP = CM::SP, PER = CM::PER;
    extern __shared__ double dsm[];
    double* sG = dsm;
    double* sT = sG + N * SP;
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    for (int e = tid; e < NN; e += kThreads)
        sG[(e / N) * SP + e % N] = S0 ? (double)S0[bh * NN + e] : ((e / N) == (e % N) ? 1.0 : 0.0);
    for (int64_t g = 0; g < p.NG; ++g) {
        const int64_t last = ((g + 1) * p.group < p.K ? (g + 1) * p.group : p.K) - 1;
        __syncthreads();
        for (int e = tid; e < NN; e += kThreads) {
            gcarry[(bh * p.NG + g) * NN + e] = sG[(e / N) * SP + e % N];
            sT[(e / N) * SP + e % N] = local[(bh * p.K + last) * NN + e];
        }
        __syncthreads();
        double acc[PER];
        CM::mul(sG, sT, acc);
        __syncthreads();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            if (!CM::valid(r)) continue;
            int row, col;
            CM::pos(r, row, col);
            sG[row * SP + col] += acc[r];
        }
    }
}

// Exclusive chunk carries: carry_k = GC_g (I + R_{g,k-1}), rounded to fp32.
template <int N>
__global__ void __launch_bounds__(kThreads)
k_carry_final(KParams p, const double* local, const double* gcarry, float* carry)
{
    constexpr int NN = N * N;
    using CM = CarryMul<N>;
    constexpr int SP = CM::SP, PER = CM::PER;
    extern __shared__ double dsm[];
    double* sG = dsm;
    double* sT = sG + N * SP;
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x / p.K, k = blockIdx.x % p.K;
    const int64_t g = k / p.group;
    const bool first = (k == g * p.group);
    for (int e = tid; e < NN; e += kThreads) {
        sG[(e / N) * SP + e % N] = gcarry[(bh * p.NG + g) * NN + e];
        sT[(e / N) * SP + e % N] = first ? 0.0 : local[(bh * p.K + k - 1) * NN + e];
    }
    __syncthreads();
    double acc[PER];
    if (!first) CM::mul(sG, sT, acc);
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        if (!CM::valid(r)) continue;
        int row, col;
        CM::pos(r, row, col);
        carry[(bh * p.K + k) * NN + row * N + col] = (float)(sG[row * SP + col] + (first ? 0.0 : acc[r]));
    }
}

// S_t = carry (I + Q_t) = carry + carry Q_t, in place; readout: o_t = carry (U + Q_t U).
template <int N>
__global__ void __launch_bounds__(kThreads)
k_fixup(KParams p, const float* carry, const float* u, int64_t snap_every, float* S_out,
        float* o_out, float* snaps)
{
    constexpr int NN = N * N;
    constexpr int PER = (NN + kThreads - 1) / kThreads;
    extern __shared__ float smem[];
    float* sC = smem;
    float* sQ = sC + NN;
    float* sCu = sQ + NN;
    const int tid = threadIdx.x;
    const int64_t chain = blockIdx.x;
    const int64_t k = chain % p.K;
    const int64_t bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    for (int e = tid; e < NN; e += kThreads) sC[e] = carry[chain * NN + e];
    __syncthreads();

    auto fix_matrix = [&](float* g) {       // g[e] <- (C + C Q)[e], Q = g
        for (int e = tid; e < NN; e += kThreads) sQ[e] = g[e];
        __syncthreads();
        float acc[PER];
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int e = tid + r * kThreads;
            if (e < NN) {
                const int i = e / N, j = e % N;
                float a = 0.0f;
#pragma unroll 8
                for (int q = 0; q < N; ++q) a = fmaf(sC[i * N + q], sQ[q * N + j], a);
                acc[r] = sC[e] + a;
            }
        }
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int e = tid + r * kThreads;
            if (e < NN) g[e] = acc[r];
        }
        __syncthreads();
    };

    if (o_out == nullptr) {
        for (int64_t t = t0; t < t1; ++t) fix_matrix(S_out + ((b * p.L + t) * p.H + h) * NN);
        return;
    }
    // readout: o_t = C U + C V_t (V_t = Q_t U, n x q) for every token of the
    // chunk, N / q tokens at a time as one small product with C transposed
    // in shared memory (thread i reads column entries C[i][j] at consecutive
    // addresses) and the V_t tile staged in sQ
    const int rq = p.rq, nq = N * rq;
    const float* uh = u + h * p.u_hs;
    float* sCt = sQ;                        // first C transposed, then reused
    for (int e = tid; e < NN; e += kThreads) sCt[(e % N) * N + e / N] = sC[e];
    __syncthreads();
    for (int e = tid; e < nq; e += kThreads) {
        const int i = e / rq, c = e - i * rq;
        float a = 0.0f;
        for (int j = 0; j < N; ++j) a = fmaf(sCt[j * N + i], uh[j * rq + c], a);
        sCu[e] = a;
    }
    __syncthreads();
    for (int e = tid; e < NN; e += kThreads) sC[e] = sCt[e];     // sC now holds C transposed
    __syncthreads();
    const int TT = N / rq;                  // tokens per tile (sQ holds TT blocks of N x q)
    float* sVt = sQ;
    for (int64_t tb = t0; tb < t1; tb += TT) {
        const int nt = (int)((t1 - tb < TT) ? t1 - tb : TT);
        for (int e = tid; e < nt * nq; e += kThreads) {
            const int tt = e / nq, r = e - tt * nq;
            sVt[e] = o_out[((b * p.L + tb + tt) * p.H + h) * nq + r];
        }
        __syncthreads();
        for (int e = tid; e < nt * nq; e += kThreads) {
            const int tt = e / nq, r = e - tt * nq, i = r / rq, c = r - i * rq;
            const float* v = sVt + tt * nq + c;
            float a = 0.0f;
#pragma unroll 8
            for (int j = 0; j < N; ++j) a = fmaf(sC[j * N + i], v[j * rq], a);
            o_out[((b * p.L + tb + tt) * p.H + h) * nq + r] = sCu[r] + a;
        }
        __syncthreads();
    }
    // snapshots need C itself again
    for (int e = tid; e < NN; e += kThreads) sQ[e] = sC[e];
    __syncthreads();
    for (int e = tid; e < NN; e += kThreads) sC[(e % N) * N + e / N] = sQ[e];
    __syncthreads();
    if (snap_every > 0) {
        const int64_t first = ((t0 + snap_every) / snap_every) * snap_every;   // 1-based
        for (int64_t t1b = first; t1b <= t1; t1b += snap_every) {
            const int64_t srow = (b * (p.L / snap_every) + t1b / snap_every - 1) * p.H + h;
            fix_matrix(snaps + srow * NN);
        }
    }
}

// ---- backward (vector-Jacobian product) -------------------------------------
//
// With G_t = dL/dS_t (every later state included): G_L = dS_L,
// G_{t-1} = dS_{t-1} + G_t X_t^T, dL/dX_t = S_{t-1}^T G_t, dL/dS0 = G_1 X_1^T
// (the chain rule of S_t = S_{t-1} X_t).  Chunked like the forward scan:
//   k_bwd_local   per chunk [t0, t1) with a zero gradient entering from the
//                 right: the local G at t0 (g_k) and W_k - I with
//                 W_k = X_{t0+1} ... X_{t1} (through the next chunk's first
//                 matrix; split form, left multiplications);
//   k_bwd_carry, or k_bwd_group / k_bwd_top / k_bwd_fix for larger
//                 problems: right to left in fp64 (serially, or in groups of
//                 about sqrt(K) chunks), the gradient entering chunk k from
//                 the right, Gin_{K-1} = 0, Gin_{k-1} = g_k + Gin_k W_k^T;
//   k_bwd_apply   per chunk: G from Gin_k down to t0 again, dX_t from the
//                 forward states, and the construction's chain rule to the
//                 embedding gradient (reshape: alpha dX; determinant-corrected:
//                 alpha c (dX - <dX, Xr> Xr^-T / n); LDU: through L, D, U).

// C = A B^T (trans) or A B of N x N matrices in shared memory, each thread
// its outputs e = tid + r * kThreads; the whole CTA calls it.
template <int N, bool BT, class Grp = CtaGroup>
__device__ __forceinline__ void cta_product(const float* A, const float* Bm, float (&acc)[(N * N + Grp::kSize - 1) / Grp::kSize])
{
    constexpr int NN = N * N;
    constexpr int PER = (NN + Grp::kSize - 1) / Grp::kSize;
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        const int e = Grp::idx() + r * Grp::kSize;
        float a = 0.0f;
        if (e < NN) {
            const int i = e / N, j = e % N;
#pragma unroll 8
            for (int k = 0; k < N; ++k) a = fmaf(A[i * N + k], BT ? Bm[j * N + k] : Bm[k * N + j], a);
        }
        acc[r] = a;
    }
}

// Xr^-1 by Gauss-Jordan elimination with partial pivoting on [sA | sI] in
// shared memory (sA destroyed, sI ends as the inverse).  The whole CTA calls
// it; sets the flag slot of sAux when a pivot column is zero.
template <int N, class Grp = CtaGroup>
__device__ void cta_inverse(float* sA, float* sI, float* sAux)
{
    constexpr int NN = N * N;
    int* sPiv = aux_piv<N>(sAux);
    for (int e = Grp::idx(); e < NN; e += Grp::kSize) sI[e] = (e / N == e % N) ? 1.0f : 0.0f;
    if (Grp::idx() == 0) *aux_flag<N>(sAux) = 0.0f;
    Grp::sync();
    for (int k = 0; k < N; ++k) {
        if (Grp::idx() < 32) {
            float best = -1.0f;
            int bi = k;
            for (int i = k + Grp::idx(); i < N; i += 32) {
                const float a = fabsf(sA[i * N + k]);
                if (a > best) { best = a; bi = i; }
            }
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_down_sync(0xffffffffu, best, o);
                const int oi = __shfl_down_sync(0xffffffffu, bi, o);
                if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            if (Grp::idx() == 0) {
                *sPiv = bi;
                if (!(best > 0.0f)) *aux_flag<N>(sAux) = 1.0f;
            }
        }
        Grp::sync();
        const int piv = *sPiv;
        if (piv != k)
            for (int j = Grp::idx(); j < N; j += Grp::kSize) {
                float a = sA[k * N + j]; sA[k * N + j] = sA[piv * N + j]; sA[piv * N + j] = a;
                a = sI[k * N + j]; sI[k * N + j] = sI[piv * N + j]; sI[piv * N + j] = a;
            }
        Grp::sync();
        const float pk = sA[k * N + k];
        const float r = (pk != 0.0f) ? 1.0f / pk : 0.0f;
        Grp::sync();
        for (int j = Grp::idx(); j < N; j += Grp::kSize) {
            sA[k * N + j] *= r;
            sI[k * N + j] *= r;
        }
        Grp::sync();
        for (int e = Grp::idx(); e < NN; e += Grp::kSize) {
            const int i = e / N, j = e % N;
            if (i == k) continue;
            const float f = sA[i * N + k];
            sI[e] = fmaf(-f, sI[k * N + j], sI[e]);
        }
        for (int e = Grp::idx(); e < NN; e += Grp::kSize) {
            const int i = e / N, j = e % N;
            if (i == k || j == k) continue;
            sA[e] = fmaf(-sA[i * N + k], sA[k * N + j], sA[e]);
        }
        Grp::sync();
        for (int i = Grp::idx(); i < N; i += Grp::kSize)
            if (i != k) sA[i * N + k] = 0.0f;
        Grp::sync();
    }
}

template <int N, class Grp>
__global__ void __launch_bounds__(kThreads)
k_bwd_local(KParams p, const void* src, const float* __restrict__ dS, float* __restrict__ gloc,
            float* __restrict__ Wq, uint32_t* status, int gfl)
{
    constexpr int NN = N * N;
    constexpr int PER = (NN + Grp::kSize - 1) / Grp::kSize;
    extern __shared__ float smem[];
    constexpr int GPB = kThreads / Grp::kSize;
    const int gi = threadIdx.x / Grp::kSize;
    const int64_t chain = (int64_t)blockIdx.x * GPB + gi;
    if (chain >= p.B * p.H * p.K) return;
    float* sG = smem + (size_t)gi * gfl;
    float* sR = sG + NN;
    float* sF = sR + NN;
    float* sM = sF + NN;
    float* sW = sM + NN;
    float* sAux = sW + NN;
    const int tid = Grp::idx();
    const int64_t k = chain % p.K, bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    const bool more = t1 < p.L;                     // a chunk follows: W_k is needed
    for (int e = tid; e < NN; e += Grp::kSize) sG[e] = dS[((b * p.L + t1 - 1) * p.H + h) * NN + e];
    if (more) {
        cta_construct<N, Grp>(p, src, ((b * p.L + t1) * p.H + h) * NN, sF, sM, sW, sAux, status);
        for (int e = tid; e < NN; e += Grp::kSize) sR[e] = sF[e];
    }
    Grp::sync();
    for (int64_t q = t1 - 1; q > t0; --q) {
        cta_construct<N, Grp>(p, src, ((b * p.L + q) * p.H + h) * NN, sF, sM, sW, sAux, status);
        float ag[PER], ar[PER];
        cta_product<N, true, Grp>(sG, sF, ag);           // G F^T
        if (more) cta_product<N, false, Grp>(sF, sR, ar);  // F R
        Grp::sync();
        const float* ds = dS + ((b * p.L + q - 1) * p.H + h) * NN;
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int e = tid + r * Grp::kSize;
            if (e < NN) {
                sG[e] = ds[e] + (sG[e] + ag[r]);     // dS_{q-1} + G X_q^T
                if (more) sR[e] = sR[e] + (sF[e] + ar[r]);    // X_q W - I
            }
        }
        Grp::sync();
    }
    for (int e = tid; e < NN; e += Grp::kSize) {
        gloc[chain * NN + e] = sG[e];
        Wq[chain * NN + e] = more ? sR[e] : 0.0f;
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes)
{
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// ---- the chunk-gradient scan, in groups --------------------------------------
//
// Chunk k's map is A_k(G) = g_k + G W_k^T (g_k = gloc_k, W_k = I + Wq_k);
// the gradient entering chunk k from the right is
// Gin_k = (A_{k+1} o ... o A_{K-1})(0).  The maps compose associatively,
// (g_a, W_a) o (g_b, W_b) = (g_a + g_b W_a^T, W_a W_b), so the right-to-left
// scan runs in groups of G chunks: k_bwd_group walks each group from its
// right end and records for every chunk the composition of the group's later
// chunks (the identity for the last) and the group's whole composition;
// k_bwd_top walks the groups from the right (the gradient entering each
// group's last chunk); k_bwd_fix applies each chunk's recorded composition
// to its group's entering gradient.  W parts in split form (W - I), all in
// fp64 (the products by CarryMul: on the fp64 tensor cores for n >= 32, W
// parts stored transposed where they multiply from the right); the serial
// steps are G + NG instead of K.

template <int N>
__global__ void __launch_bounds__(kThreads)
k_bwd_group(KParams p, const float* __restrict__ gloc, const float* __restrict__ Wq, int gshift, int64_t NG,
            double* __restrict__ sg, double* __restrict__ sw, double* __restrict__ gg, double* __restrict__ gw)
{
    constexpr int NN = N * N;
    using CM = CarryMul<N>;
    constexpr int SP = CM::SP, PER = CM::PER;
    extern __shared__ double dsm[];
    double* cg = dsm;                       // the running composition's g part
    double* cw = cg + N * SP;               // its W part, W - I
    double* sq = cw + N * SP;               // Q_k = W_k - I of the chunk at hand
    double* sqt = sq + N * SP;              // Q_k^T
    const int tid = threadIdx.x;
    const int64_t seq = blockIdx.x / NG, grp = blockIdx.x - seq * NG;
    const int64_t k0 = grp << gshift;
    const int64_t k1 = (k0 + ((int64_t)1 << gshift) < p.K) ? k0 + ((int64_t)1 << gshift) : p.K;
    for (int e = tid; e < N * SP; e += kThreads) {
        cg[e] = 0.0;
        cw[e] = 0.0;
    }
    __syncthreads();
    for (int64_t k = k1 - 1; k >= k0; --k) {
        const int64_t chain = seq * p.K + k;
        for (int e = tid; e < NN; e += kThreads) {
            const int i = e / N, j = e % N;
            sg[chain * NN + e] = cg[i * SP + j];
            sw[chain * NN + e] = cw[i * SP + j];
            const double qv = (double)Wq[chain * NN + e];
            sq[i * SP + j] = qv;
            sqt[j * SP + i] = qv;
        }
        __syncthreads();
        double ag[PER], aw[PER];
        CM::mul(cg, sqt, ag);               // cg Q^T
        CM::mul(sq, cw, aw);                // Q cw
        __syncthreads();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            if (!CM::valid(r)) continue;
            int row, col;
            CM::pos(r, row, col);
            const int e = row * SP + col;
            cg[e] = (double)gloc[chain * NN + row * N + col] + (cg[e] + ag[r]);   // g_k + cg (I + Q)^T
            cw[e] = sq[e] + (cw[e] + aw[r]);                                       // (I + Q)(I + cw) - I
        }
        __syncthreads();
    }
    for (int e = tid; e < NN; e += kThreads) {
        const int i = e / N, j = e % N;
        gg[blockIdx.x * (int64_t)NN + e] = cg[i * SP + j];
        gw[blockIdx.x * (int64_t)NN + e] = cw[i * SP + j];
    }
}

template <int N>
__global__ void __launch_bounds__(kThreads)
k_bwd_top(int64_t NG, const double* __restrict__ gg, const double* __restrict__ gw, double* __restrict__ ginr)
{
    constexpr int NN = N * N;
    using CM = CarryMul<N>;
    constexpr int SP = CM::SP, PER = CM::PER;
    extern __shared__ double dsm[];
    double* cur = dsm;
    double* wt = cur + N * SP;              // (W_G - I)^T of the group at hand
    const int tid = threadIdx.x;
    const int64_t base = (int64_t)blockIdx.x * NG;
    for (int e = tid; e < N * SP; e += kThreads) cur[e] = 0.0;
    __syncthreads();
    for (int64_t grp = NG - 1; grp >= 0; --grp) {
        const int64_t gi = (base + grp) * NN;
        for (int e = tid; e < NN; e += kThreads) {
            const int i = e / N, j = e % N;
            ginr[gi + e] = cur[i * SP + j];
            wt[j * SP + i] = gw[gi + e];
        }
        __syncthreads();
        double acc[PER];
        CM::mul(cur, wt, acc);              // cur W_G^T (split)
        __syncthreads();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            if (!CM::valid(r)) continue;
            int row, col;
            CM::pos(r, row, col);
            cur[row * SP + col] = gg[gi + row * N + col] + (cur[row * SP + col] + acc[r]);
        }
        __syncthreads();
    }
}

template <int N>
__global__ void __launch_bounds__(kThreads)
k_bwd_fix(KParams p, int gshift, int64_t NG, const double* __restrict__ sg, const double* __restrict__ sw,
          const double* __restrict__ ginr, float* __restrict__ Gin)
{
    constexpr int NN = N * N;
    using CM = CarryMul<N>;
    constexpr int SP = CM::SP, PER = CM::PER;
    extern __shared__ double dsm[];
    double* gr = dsm;
    double* wt = gr + N * SP;
    const int tid = threadIdx.x;
    const int64_t chain = blockIdx.x;
    const int64_t seq = chain / p.K, k = chain - seq * p.K;
    const int64_t gi = (seq * NG + (k >> gshift)) * NN;
    for (int e = tid; e < NN; e += kThreads) {
        const int i = e / N, j = e % N;
        gr[i * SP + j] = ginr[gi + e];
        wt[j * SP + i] = sw[chain * NN + e];
    }
    __syncthreads();
    double acc[PER];
    CM::mul(gr, wt, acc);                   // Ginr W_suf^T (split)
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        if (!CM::valid(r)) continue;
        int row, col;
        CM::pos(r, row, col);
        const int64_t e = chain * NN + row * N + col;
        Gin[e] = (float)(sg[e] + (gr[row * SP + col] + acc[r]));
    }
}

// The same scan serially, one CTA per sequence right to left (fewer
// launches and no per-chunk records: the choice for small problems).
template <int N>
__global__ void __launch_bounds__(kThreads)
k_bwd_carry(KParams p, const float* __restrict__ gloc, const float* __restrict__ Wq, float* __restrict__ Gin)
{
    constexpr int NN = N * N;
    using CM = CarryMul<N>;
    constexpr int SP = CM::SP, PER = CM::PER;
    extern __shared__ double dsm[];
    double* sGin = dsm;
    double* sWt = sGin + N * SP;            // (W_k - I)^T
    const int tid = threadIdx.x;
    const int64_t seq = blockIdx.x;
    for (int e = tid; e < N * SP; e += kThreads) sGin[e] = 0.0;
    __syncthreads();
    for (int64_t k = p.K - 1; k >= 0; --k) {
        const int64_t chain = seq * p.K + k;
        for (int e = tid; e < NN; e += kThreads) {
            const int i = e / N, j = e % N;
            Gin[chain * NN + e] = (float)sGin[i * SP + j];
            sWt[j * SP + i] = (double)Wq[chain * NN + e];
        }
        __syncthreads();
        if (k == 0) break;
        double acc[PER];
        CM::mul(sGin, sWt, acc);            // Gin Wq^T
        __syncthreads();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            if (!CM::valid(r)) continue;
            int row, col;
            CM::pos(r, row, col);
            sGin[row * SP + col] = (double)gloc[chain * NN + row * N + col] + (sGin[row * SP + col] + acc[r]);
        }
        __syncthreads();
    }
}

// The chunk-gradient scan: Gin from gloc, Wq.  Serially per sequence while
// K n^3 is at most 2^20 (measured on B200: B8 H8 L4096, n = 16, K = 128 takes
// 0.082 ms serially, 0.105 ms in groups), else in groups (B1 H8 L262144,
// n = 16: 0.63 ms serially, 0.14 ms in groups; n = 32, K = 128: 0.33 and
// 0.27 ms).
template <int N>
cudaError_t bwd_carry_scan(const KParams& p, const float* gloc, const float* Wq, float* Gin, char* ws,
                           const BwdWorkspace& W, cudaStream_t s)
{
    const int64_t BH = p.B * p.H, chains = BH * p.K;
    if (chains == 0) return cudaSuccess;
    constexpr int SP = CarryMul<N>::SP;
    if (p.K * (int64_t)N * N * N <= ((int64_t)1 << 20)) {
        const size_t sm_carry = sizeof(double) * 2 * N * SP;
        cudaError_t e = set_smem(k_bwd_carry<N>, sm_carry);
        if (e != cudaSuccess) return e;
        k_bwd_carry<N><<<(unsigned)BH, kThreads, sm_carry, s>>>(p, gloc, Wq, Gin);
        return cudaGetLastError();
    }
    double* sg = reinterpret_cast<double*>(ws + W.sg);
    double* sw = reinterpret_cast<double*>(ws + W.sw);
    double* gg = reinterpret_cast<double*>(ws + W.gg);
    double* gw = reinterpret_cast<double*>(ws + W.gw);
    double* ginr = reinterpret_cast<double*>(ws + W.ginr);
    const size_t sm3 = sizeof(double) * 4 * N * SP, sm2 = sizeof(double) * 2 * N * SP;
    cudaError_t e;
    if ((e = set_smem(k_bwd_group<N>, sm3)) != cudaSuccess) return e;
    if ((e = set_smem(k_bwd_top<N>, sm2)) != cudaSuccess) return e;
    if ((e = set_smem(k_bwd_fix<N>, sm2)) != cudaSuccess) return e;
    k_bwd_group<N><<<(unsigned)(BH * W.NG), kThreads, sm3, s>>>(p, gloc, Wq, W.gshift, W.NG, sg, sw, gg, gw);
    k_bwd_top<N><<<(unsigned)BH, kThreads, sm2, s>>>(W.NG, gg, gw, ginr);
    k_bwd_fix<N><<<(unsigned)chains, kThreads, sm2, s>>>(p, W.gshift, W.NG, sg, sw, ginr, Gin);
    return cudaGetLastError();
}

// dA = L(A^T, dX), the adjoint of the Frechet derivative of exp at A (the
// derivative at A^T), for A = alpha (M - M^T) / 2 of the slice at src + off;
// with C = A^T = -A: B = C / 2^s, the Taylor part differentiates Horner's
// recurrence (Y_k = B (I + Y_{k+1}) / k, so
// dY_k = (E (I + Y_{k+1}) + B dY_{k+1}) / k with E = dX / 2^s, dY_m = E / m),
// and every squaring X' = X X adds L' = X L + L X = 2L + Y L + L Y (X = I + Y).
// The same s and m as the forward.  dX comes in sD, dA goes out in sD;
// sM, sW, sS, sA, sX and sAux are scratch.  The whole CTA calls it.
template <int N, class Grp = CtaGroup>
__device__ void expm_vjp(const KParams& p, const void* src, int64_t off, float* sD, float* sM, float* sW,
                         float* sS, float* sA, float* sX, float* sAux)
{
    constexpr int NN = N * N;
    const int tid = Grp::idx();
    for (int e = tid; e < NN; e += Grp::kSize) sM[e] = load_elem(src, off + e, p.x_dtype);
    Grp::sync();
    const float ha = 0.5f * p.alpha;
    for (int e = tid; e < NN; e += Grp::kSize) {
        const int i = e / N, j = e % N;
        sA[e] = ha * (sM[j * N + i] - sM[e]);                 // C = A^T
    }
    Grp::sync();
    int m, sq;
    expm_plan<N, Grp>(sA, sAux, m, sq);
    const float scale = ldexpf(1.0f, -sq);
    float* B = sA;
    float* E = sM;
    float* Y = sW;
    float* Yn = sS;
    float* dY = sD;
    float* dYn = sX;
    for (int e = tid; e < NN; e += Grp::kSize) {
        B[e] *= scale;
        E[e] = sD[e] * scale;
    }
    Grp::sync();
    const float rm = 1.0f / (float)m;
    for (int e = tid; e < NN; e += Grp::kSize) {
        Y[e] = B[e] * rm;
        dY[e] = E[e] * rm;
    }
    Grp::sync();
    for (int k = m - 1; k >= 1; --k) {
        const float rk = 1.0f / (float)k;
        for (int e = tid; e < NN; e += Grp::kSize) {
            const int i = e / N, j = e % N;
            float a1 = 0.0f, a2 = 0.0f;
#pragma unroll 4
            for (int q = 0; q < N; ++q) {
                const float y = Y[q * N + j];
                a1 = fmaf(B[i * N + q], y, a1);
                a2 = fmaf(E[i * N + q], y, a2);
                a2 = fmaf(B[i * N + q], dY[q * N + j], a2);
            }
            Yn[e] = (B[e] + a1) * rk;
            dYn[e] = (E[e] + a2) * rk;
        }
        Grp::sync();
        float* t = Y; Y = Yn; Yn = t;
        t = dY; dY = dYn; dYn = t;
    }
    for (int r = 0; r < sq; ++r) {
        for (int e = tid; e < NN; e += Grp::kSize) {
            const int i = e / N, j = e % N;
            float a1 = 0.0f, a2 = 0.0f;
#pragma unroll 4
            for (int q = 0; q < N; ++q) {
                a1 = fmaf(Y[i * N + q], Y[q * N + j], a1);
                a2 = fmaf(Y[i * N + q], dY[q * N + j], a2);
                a2 = fmaf(dY[i * N + q], Y[q * N + j], a2);
            }
            Yn[e] = 2.0f * Y[e] + a1;
            dYn[e] = 2.0f * dY[e] + a2;
        }
        Grp::sync();
        float* t = Y; Y = Yn; Yn = t;
        t = dY; dY = dYn; dYn = t;
    }
    if (dY != sD) {
        for (int e = tid; e < NN; e += Grp::kSize) sD[e] = dY[e];
        Grp::sync();
    }
}

template <int N, class Grp>
__global__ void __launch_bounds__(kThreads)
k_bwd_apply(KParams p, const void* src, const float* __restrict__ S0, const float* __restrict__ S_fwd,
            const float* __restrict__ dS, const float* __restrict__ Gin, float* __restrict__ dx,
            float* __restrict__ dS0, uint32_t* status, int gfl)
{
    constexpr int NN = N * N;
    constexpr int PER = (NN + Grp::kSize - 1) / Grp::kSize;
    extern __shared__ float smem[];
    constexpr int GPB = kThreads / Grp::kSize;
    const int gi = threadIdx.x / Grp::kSize;
    const int64_t chain = (int64_t)blockIdx.x * GPB + gi;
    if (chain >= p.B * p.H * p.K) return;
    float* sG = smem + (size_t)gi * gfl;
    float* sF = sG + NN;
    float* sM = sF + NN;
    float* sW = sM + NN;
    float* sS = sW + NN;
    float* sD = sS + NN;
    float* sA = sD + NN;
    float* sX = sA + NN;
    float* sAux = sX + NN;
    float* sRed = sAux + 4 * N + 8;                 // Grp::kSize / 32 partial sums
    const int tid = Grp::idx();
    const int64_t k = chain % p.K, bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    for (int e = tid; e < NN; e += Grp::kSize) sG[e] = dS[((b * p.L + t1 - 1) * p.H + h) * NN + e];
    if (t1 < p.L) {
        // G_{t1-1} = dS_{t1-1} + Gin X_{t1}^T with X_{t1} = I + F
        cta_construct<N, Grp>(p, src, ((b * p.L + t1) * p.H + h) * NN, sF, sM, sW, sAux, status);
        for (int e = tid; e < NN; e += Grp::kSize) sS[e] = Gin[chain * NN + e];
        Grp::sync();
        float ag[PER];
        cta_product<N, true, Grp>(sS, sF, ag);
        Grp::sync();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int e = tid + r * Grp::kSize;
            if (e < NN) sG[e] += sS[e] + ag[r];
        }
    }
    Grp::sync();
    for (int64_t t = t1 - 1; t >= t0; --t) {
        const int64_t row = (b * p.L + t) * p.H + h;
        cta_construct<N, Grp>(p, src, row * NN, sF, sM, sW, sAux, status);
        // S_{t-1} (the state before this token)
        for (int e = tid; e < NN; e += Grp::kSize) {
            float v;
            if (t > 0) v = S_fwd[((b * p.L + t - 1) * p.H + h) * NN + e];
            else v = S0 ? S0[bh * NN + e] : ((e / N == e % N) ? 1.0f : 0.0f);
            sS[e] = v;
        }
        Grp::sync();
        // dX = S_{t-1}^T G
        {
            float acc[PER];
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                const int e = tid + r * Grp::kSize;
                float a = 0.0f;
                if (e < NN) {
                    const int i = e / N, j = e % N;
#pragma unroll 8
                    for (int q = 0; q < N; ++q) a = fmaf(sS[q * N + i], sG[q * N + j], a);
                }
                acc[r] = a;
            }
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                const int e = tid + r * Grp::kSize;
                if (e < NN) sD[e] = acc[r];
            }
        }
        Grp::sync();
        float* out = dx + row * NN;
        if (p.mode == MRU_MODE_RESHAPE) {
            for (int e = tid; e < NN; e += Grp::kSize) out[e] = p.alpha * sD[e];
        } else if (p.mode == MRU_MODE_DETNORM) {
            // dXr = c (dX - <dX, Xr> Xr^-T / N), dM = alpha dXr
            const float c = aux_c<N>(sAux)[0];
            float part = 0.0f;
            for (int e = tid; e < NN; e += Grp::kSize) {
                float xr = p.alpha * sM[e];
                if (p.add_identity && e / N == e % N) xr += 1.0f;
                sA[e] = xr;
                part = fmaf(sD[e], xr, part);
            }
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            float inner = part;                   // one warp: every lane has the sum
            if constexpr (Grp::kSize > 32) {
                if ((tid & 31) == 0) sRed[tid >> 5] = part;
                Grp::sync();
                inner = 0.0f;
                for (int w = 0; w < Grp::kSize / 32; ++w) inner += sRed[w];
            }
            cta_inverse<N, Grp>(sA, sW, sAux);             // sW = Xr^-1
            const float f = inner / N;
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                out[e] = (c == 0.0f) ? 0.0f : p.alpha * c * fmaf(-f, sW[j * N + i], sD[e]);
            }
        } else if (p.mode == MRU_MODE_CAYLEY) {
            // X = 2 W^-1 - I with W = I - A, so W^-1 = I + F / 2 and
            // dA = 2 W^-T dX W^-T = 2 T + T F^T with T = dX + F^T dX / 2
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                float a = 0.0f;
#pragma unroll 8
                for (int q = 0; q < N; ++q) a = fmaf(sF[q * N + i], sD[q * N + j], a);
                sA[e] = fmaf(0.5f, a, sD[e]);
            }
            Grp::sync();
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                float a = 0.0f;
#pragma unroll 8
                for (int q = 0; q < N; ++q) a = fmaf(sA[i * N + q], sF[j * N + q], a);
                sS[e] = 2.0f * sA[e] + a;
            }
            Grp::sync();
            const float ha = 0.5f * p.alpha;       // A = alpha (M - M^T) / 2
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                out[e] = ha * (sS[e] - sS[j * N + i]);
            }
        } else if (p.mode == MRU_MODE_EXPM) {
            expm_vjp<N, Grp>(p, src, row * NN, sD, sM, sW, sS, sA, sX, sAux);   // dA in sD
            const float ha = 0.5f * p.alpha;
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                out[e] = ha * (sD[e] - sD[j * N + i]);
            }
        } else {
            // LDU: D_i = sAux[i] (and D_i - 1 = sAux[N + i]) from the construction
            const float a = p.ldu_a;
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                float v;
                if (i > j) {
                    // dL_ij = sum_{q >= j} dX_iq D_j U_jq (U_jj = 1)
                    float s2 = sD[i * N + j];
                    for (int q = j + 1; q < N; ++q) s2 = fmaf(sD[i * N + q], a * sM[j * N + q], s2);
                    v = a * sAux[j] * s2;
                } else {
                    // d(DU)_ij = sum_{q >= i} L_qi dX_qj (L_ii = 1)
                    float s2 = sD[i * N + j];
                    for (int q = i + 1; q < N; ++q) s2 = fmaf(a * sM[q * N + i], sD[q * N + j], s2);
                    v = (i < j) ? a * sAux[i] * s2 : s2;   // diagonal: d(DU)_ii, finished below
                }
                sA[e] = v;
            }
            Grp::sync();
            for (int e = tid; e < NN; e += Grp::kSize) {
                const int i = e / N, j = e % N;
                if (i != j) { out[e] = sA[e]; continue; }
                // dD_i = sum_j d(DU)_ij U_ij = d(DU)_ii + sum_{j > i} (dM_ij / (a D_i)) a M_ij
                float dD = sA[e];
                for (int q = i + 1; q < N; ++q) {
                    // d(DU)_iq = dM_iq / (a D_i)
                    float s2 = sD[i * N + q];
                    for (int r2 = i + 1; r2 < N; ++r2) s2 = fmaf(a * sM[r2 * N + i], sD[r2 * N + q], s2);
                    dD = fmaf(s2, a * sM[i * N + q], dD);
                }
                const float th = tanhf(sM[e]);
                out[e] = dD * sAux[i] * p.ldu_d * (1.0f - th * th);
            }
        }
        Grp::sync();
        // dS0 = G X_1^T, or G_{t-1} = dS_{t-1} + G X_t^T
        float ag[PER];
        cta_product<N, true, Grp>(sG, sF, ag);
        Grp::sync();
        if (t == 0) {
            if (dS0)
#pragma unroll
                for (int r = 0; r < PER; ++r) {
                    const int e = tid + r * Grp::kSize;
                    if (e < NN) dS0[bh * NN + e] = sG[e] + ag[r];
                }
        } else if (t > t0) {
            const float* ds = dS + ((b * p.L + t - 1) * p.H + h) * NN;
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                const int e = tid + r * Grp::kSize;
                if (e < NN) sG[e] = ds[e] + (sG[e] + ag[r]);
            }
        }
        Grp::sync();
    }
}

template <int N>
cudaError_t backward_n(const KParams& p, const void* src, const float* S0, const float* S_fwd, const float* dS,
                       float* dx, float* dS0, char* ws, const BwdWorkspace& W, cudaStream_t s);


template <int N>
cudaError_t backward_n(const KParams& p, const void* src, const float* S0, const float* S_fwd, const float* dS,
                       float* dx, float* dS0, char* ws, const BwdWorkspace& W, cudaStream_t s)
{
    constexpr int NN = N * N;
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + W.status);
    float* gloc = reinterpret_cast<float*>(ws + W.gloc);
    float* Wq = reinterpret_cast<float*>(ws + W.wq);
    float* Gin = reinterpret_cast<float*>(ws + W.gin);
    const int64_t BH = p.B * p.H;
    const int64_t chains = BH * p.K;
    if (chains == 0) return cudaSuccess;
    cudaError_t e;
    // n <= 16: one warp per chunk (eight per CTA, __syncwarp only); larger n:
    // one CTA per chunk
    using Grp = typename std::conditional<(N <= 16), WarpGroup, CtaGroup>::type;
    constexpr int GPB = kThreads / Grp::kSize;
    const int gfl_local = 5 * NN + 4 * N + 8;
    const int gfl_apply = 8 * NN + 4 * N + 8 + kThreads / 32;
    const size_t sm_local = sizeof(float) * gfl_local * GPB;
    const size_t sm_apply = sizeof(float) * gfl_apply * GPB;
    const unsigned grid = (unsigned)((chains + GPB - 1) / GPB);
    if (N == 16 && n16::supports_backward(p)) {
        // n = 16 on the tensor cores; the chunk-gradient scan stays generic
        const float* x = reinterpret_cast<const float*>(src);
        profile_mark(0, 0, s);
        if ((e = n16::launch_bwd_local(p, x, dS, gloc, Wq, status, s)) != cudaSuccess) return e;
        profile_mark(0, 1, s);
        profile_mark(1, 0, s);
        if ((e = bwd_carry_scan<N>(p, gloc, Wq, Gin, ws, W, s)) != cudaSuccess) return e;
        profile_mark(1, 1, s);
        profile_mark(2, 0, s);
        if ((e = n16::launch_bwd_apply(p, x, S0, S_fwd, dS, Gin, dx, dS0, status, s)) != cudaSuccess) return e;
        profile_mark(2, 1, s);
        return cudaGetLastError();
    }
    if (N == 32 && n32::supports_backward(p)) {
        // n = 32 LDU on the tensor cores; the chunk-gradient scan stays generic
        profile_mark(0, 0, s);
        if ((e = n32::launch_bwd_local(p, src, dS, gloc, Wq, s)) != cudaSuccess) return e;
        profile_mark(0, 1, s);
        profile_mark(1, 0, s);
        if ((e = bwd_carry_scan<N>(p, gloc, Wq, Gin, ws, W, s)) != cudaSuccess) return e;
        profile_mark(1, 1, s);
        profile_mark(2, 0, s);
        if ((e = n32::launch_bwd_apply(p, src, S0, S_fwd, dS, Gin, dx, dS0, s)) != cudaSuccess) return e;
        profile_mark(2, 1, s);
        return cudaGetLastError();
    }
    if (N == 64 && n64::supports_backward(p)) {
        // n = 64 in tf32 on the tensor cores; the chunk-gradient scan stays generic
        const float* x = reinterpret_cast<const float*>(src);
        profile_mark(0, 0, s);
        if ((e = n64::launch_bwd_local(p, x, dS, gloc, Wq, status, s)) != cudaSuccess) return e;
        profile_mark(0, 1, s);
        profile_mark(1, 0, s);
        if ((e = bwd_carry_scan<N>(p, gloc, Wq, Gin, ws, W, s)) != cudaSuccess) return e;
        profile_mark(1, 1, s);
        profile_mark(2, 0, s);
        if ((e = n64::launch_bwd_apply(p, x, S0, S_fwd, dS, Gin, dx, dS0, status, s)) != cudaSuccess) return e;
        profile_mark(2, 1, s);
        return cudaGetLastError();
    }
    if ((e = set_smem(k_bwd_local<N, Grp>, sm_local)) != cudaSuccess) return e;
    if ((e = set_smem(k_bwd_apply<N, Grp>, sm_apply)) != cudaSuccess) return e;
    profile_mark(0, 0, s);
    k_bwd_local<N, Grp><<<grid, kThreads, sm_local, s>>>(p, src, dS, gloc, Wq, status, gfl_local);
    profile_mark(0, 1, s);
    profile_mark(1, 0, s);
    if ((e = bwd_carry_scan<N>(p, gloc, Wq, Gin, ws, W, s)) != cudaSuccess) return e;
    profile_mark(1, 1, s);
    profile_mark(2, 0, s);
    k_bwd_apply<N, Grp><<<grid, kThreads, sm_apply, s>>>(p, src, S0, S_fwd, dS, Gin, dx, dS0, status, gfl_apply);
    profile_mark(2, 1, s);
    return cudaGetLastError();
}

template <int N>
cudaError_t build_states_n(const KParams& p, const void* x, float* X_out, int smi, uint32_t* status,
                           cudaStream_t s)
{
    constexpr int NN = N * N;
    const size_t sm = sizeof(float) * (3 * NN + 4 * N + 8);
    cudaError_t e = set_smem(k_build_states<N>, sm);
    if (e != cudaSuccess) return e;
    const int64_t rows = p.B * p.L * p.H;
    const int64_t grid = rows < 148 * 64 ? rows : 148 * 64;
    if (grid > 0) k_build_states<N><<<(unsigned)grid, kThreads, sm, s>>>(p, x, X_out, smi, status);
    return cudaGetLastError();
}

// ---- small problems in one launch (n = 4, the whole sequence one chunk) ------
//
// One CTA per sequence; thread i takes the tokens [i T, (i + 1) T) with
// T = ceil(L / 256), forms their product in registers (fp64), the CTA scans
// the 256 products in fp64 (shuffles within each warp, then the eight warp
// totals), and every thread re-runs its tokens in fp32 from its exclusive
// carry S0 P_0 ... P_{i-1}, writing S_t.  The construction
// follows cta_construct's arithmetic token by token in the thread.

constexpr int SN = 4, SNN = SN * SN;

// The 16 values of one token (its embedding slice, or X or F for lifted
// input) as fp32, in 16-byte loads: the boundary takes 16-byte aligned
// buffers only and a token starts at a multiple of 16 elements.
__device__ __forceinline__ void small_load(const KParams& p, const void* src, int64_t off, float (&M)[SNN])
{
    if (p.src == SRC_EMBEDDING && p.x_dtype == MRU_BF16) {
        const uint4* q = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(src) + off);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint4 v = __ldg(q + r);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {      // element 2k in the low half of word k
                M[8 * r + 2 * k] = __uint_as_float(w[k] << 16);
                M[8 * r + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
            }
        }
        return;
    }
    const float4* q = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + off);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float4 v = __ldg(q + r);
        M[4 * r] = v.x; M[4 * r + 1] = v.y; M[4 * r + 2] = v.z; M[4 * r + 3] = v.w;
    }
}

// F = X - I of one token from its loaded values M.  Returns false for a
// singular determinant-corrected matrix (F is then 0: X = I, output
// unspecified).
__device__ __forceinline__ bool small_construct(const KParams& p, const float (&M)[SNN], float (&F)[SNN])
{
    if (p.src != SRC_EMBEDDING) {
#pragma unroll
        for (int e = 0; e < SNN; ++e) F[e] = M[e] - ((p.src == SRC_X && e / SN == e % SN) ? 1.0f : 0.0f);
        return true;
    }
    if (p.mode == MRU_MODE_RESHAPE) {
#pragma unroll
        for (int e = 0; e < SNN; ++e) F[e] = p.alpha * M[e] - ((!p.add_identity && e / SN == e % SN) ? 1.0f : 0.0f);
        return true;
    }
    if (p.mode == MRU_MODE_LDU) {
        float D[SN], Dm1[SN];
#pragma unroll
        for (int k = 0; k < SN; ++k) {
            const double z = (double)p.ldu_d * tanh((double)M[k * SN + k]);
            D[k] = (float)exp(z);
            Dm1[k] = (float)expm1(z);
        }
        const float a = p.ldu_a;
#pragma unroll
        for (int i = 0; i < SN; ++i)
#pragma unroll
            for (int j = 0; j < SN; ++j) {
                const int m = i < j ? i : j;
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < m; ++k) acc = fmaf(a * M[i * SN + k] * D[k], a * M[k * SN + j], acc);
                if (i < j) acc = fmaf(D[i], a * M[i * SN + j], acc);
                else if (i > j) acc = fmaf(a * M[i * SN + j], D[j], acc);
                else acc += Dm1[i];
                F[i * SN + j] = acc;
            }
        return true;
    }
    // determinant-corrected: X = c Xr, c = |det Xr|^(-1/n)
    double ld = 0.0;
    bool pivot = !p.add_identity, singular = false;
    if (p.add_identity) {                       // near the identity: eliminate E alone
        float W[SNN];
#pragma unroll
        for (int e = 0; e < SNN; ++e) W[e] = p.alpha * M[e];
        double prod = 1.0;
#pragma unroll
        for (int k = 0; k < SN; ++k) {
            const float d = W[k * SN + k];
            if (!(fabsf(1.0f + d) >= 0.5f)) pivot = true;
            prod *= 1.0 + (double)d;
            const float r = 1.0f / (1.0f + d);
#pragma unroll
            for (int i = k + 1; i < SN; ++i)
#pragma unroll
                for (int j = k + 1; j < SN; ++j) W[i * SN + j] = fmaf(-W[i * SN + k] * r, W[k * SN + j], W[i * SN + j]);
        }
        ld = log(fabs(prod));
    }
    if (pivot) {                                // partial pivoting on Xr itself
        float W[SNN];
#pragma unroll
        for (int e = 0; e < SNN; ++e) W[e] = p.alpha * M[e] + ((p.add_identity && e / SN == e % SN) ? 1.0f : 0.0f);
        ld = 0.0;
#pragma unroll
        for (int k = 0; k < SN; ++k) {
            int piv = k;
            float best = fabsf(W[k * SN + k]);
#pragma unroll
            for (int i = k + 1; i < SN; ++i)
                if (fabsf(W[i * SN + k]) > best) { best = fabsf(W[i * SN + k]); piv = i; }
            if (!(best > 0.0f)) singular = true;
#pragma unroll
            for (int i = k + 1; i < SN; ++i)   // swap rows k and piv (compile-time registers, selects)
                if (i == piv)
#pragma unroll
                    for (int j = 0; j < SN; ++j) {
                        const float tmp = W[k * SN + j];
                        W[k * SN + j] = W[i * SN + j];
                        W[i * SN + j] = tmp;
                    }
            const float pk = W[k * SN + k];
            ld += log(fabs((double)pk));
            const float r = pk != 0.0f ? 1.0f / pk : 0.0f;
#pragma unroll
            for (int i = k + 1; i < SN; ++i)
#pragma unroll
                for (int j = k + 1; j < SN; ++j) W[i * SN + j] = fmaf(-W[i * SN + k] * r, W[k * SN + j], W[i * SN + j]);
        }
    }
    const double cm1 = expm1(-ld / SN);
    float c = (float)(1.0 + cm1), cm1f = (float)cm1;
    if (singular || !isfinite(ld) || !isfinite(c) || c == 0.0f) {
#pragma unroll
        for (int e = 0; e < SNN; ++e) F[e] = 0.0f;
        return false;
    }
#pragma unroll
    for (int e = 0; e < SNN; ++e)
        F[e] = c * (p.alpha * M[e]) + ((e / SN == e % SN) ? (p.add_identity ? cm1f : -1.0f) : 0.0f);
    return true;
}

__device__ __forceinline__ void d4_mul(const double (&A)[SNN], const double (&B)[SNN], double (&C)[SNN])
{
#pragma unroll
    for (int i = 0; i < SN; ++i)
#pragma unroll
        for (int j = 0; j < SN; ++j) {
            double a = 0.0;
#pragma unroll
            for (int k = 0; k < SN; ++k) a = fma(A[i * SN + k], B[k * SN + j], a);
            C[i * SN + j] = a;
        }
}

__global__ void __launch_bounds__(kThreads)
k_small_scan(KParams p, const void* src, float* __restrict__ S_out, const float* __restrict__ S0, uint32_t* status)
{
    __shared__ double wtot[kThreads / 32][SNN];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.x, h = bh % p.H, b = bh / p.H;
    const int64_t T = (p.L + kThreads - 1) / kThreads;
    const int64_t t0 = tid * T < p.L ? tid * T : p.L, t1 = t0 + T < p.L ? t0 + T : p.L;
    bool bad = false;
    // tokens are loaded two ahead of their use (ring of three)
    const int64_t stride = p.H * SNN, base = (b * p.L * p.H + h) * SNN;
    float M0[SNN] = {}, M1[SNN] = {};
    if (t0 < t1) small_load(p, src, base + t0 * stride, M0);
    if (t0 + 1 < t1) small_load(p, src, base + (t0 + 1) * stride, M1);
    // segment product in fp64, P <- P + P F, so that the carries hold little
    // more than the rounding of each token's F (fp32 segment products gave
    // 3.5x the worst-token error on rotated near-permutation chains)
    double P[SNN];
#pragma unroll
    for (int e = 0; e < SNN; ++e) P[e] = (e / SN == e % SN) ? 1.0 : 0.0;
    for (int64_t t = t0; t < t1; ++t) {
        float M2[SNN] = {};
        if (t + 2 < t1) small_load(p, src, base + (t + 2) * stride, M2);
        float F[SNN];
        bad |= !small_construct(p, M0, F);
#pragma unroll
        for (int e = 0; e < SNN; ++e) { M0[e] = M1[e]; M1[e] = M2[e]; }
        double PF[SNN];
#pragma unroll
        for (int i = 0; i < SN; ++i)
#pragma unroll
            for (int j = 0; j < SN; ++j) {
                double a = P[i * SN + j];
#pragma unroll
                for (int k = 0; k < SN; ++k) a = fma(P[i * SN + k], (double)F[k * SN + j], a);
                PF[i * SN + j] = a;
            }
#pragma unroll
        for (int e = 0; e < SNN; ++e) P[e] = PF[e];
    }
    if (bad) atomicOr(status, STATUS_SINGULAR);
    // inclusive scan of the segment products over the warp, fp64, in order
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        double O[SNN], R[SNN];
#pragma unroll
        for (int e = 0; e < SNN; ++e) O[e] = __shfl_up_sync(0xffffffffu, P[e], d);
        d4_mul(O, P, R);
        if (lane >= d) {
#pragma unroll
            for (int e = 0; e < SNN; ++e) P[e] = R[e];
        }
    }
    if (lane == 31) {
#pragma unroll
        for (int e = 0; e < SNN; ++e) wtot[warp][e] = P[e];
    }
    __syncthreads();
    // exclusive carry: S0 (or I), the earlier warps' totals, this warp's lanes before
    double C[SNN], R[SNN];
#pragma unroll
    for (int e = 0; e < SNN; ++e) C[e] = S0 ? (double)S0[bh * SNN + e] : ((e / SN == e % SN) ? 1.0 : 0.0);
    for (int w = 0; w < warp; ++w) {
        double Wt[SNN];
#pragma unroll
        for (int e = 0; e < SNN; ++e) Wt[e] = wtot[w][e];
        d4_mul(C, Wt, R);
#pragma unroll
        for (int e = 0; e < SNN; ++e) C[e] = R[e];
    }
    {
        double O[SNN];
#pragma unroll
        for (int e = 0; e < SNN; ++e) O[e] = __shfl_up_sync(0xffffffffu, P[e], 1);
        if (lane > 0) {
            d4_mul(C, O, R);
#pragma unroll
            for (int e = 0; e < SNN; ++e) C[e] = R[e];
        }
    }
    // re-run from the carry: S <- S + S F, every S_t written
    float S[SNN];
#pragma unroll
    for (int e = 0; e < SNN; ++e) S[e] = (float)C[e];
    if (t0 < t1) small_load(p, src, base + t0 * stride, M0);
    if (t0 + 1 < t1) small_load(p, src, base + (t0 + 1) * stride, M1);
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t row = base + t * stride;
        float M2[SNN] = {};
        if (t + 2 < t1) small_load(p, src, base + (t + 2) * stride, M2);
        float F[SNN];
        small_construct(p, M0, F);
#pragma unroll
        for (int e = 0; e < SNN; ++e) { M0[e] = M1[e]; M1[e] = M2[e]; }
        float SF[SNN];
#pragma unroll
        for (int i = 0; i < SN; ++i)
#pragma unroll
            for (int j = 0; j < SN; ++j) {
                float a = 0.0f;
#pragma unroll
                for (int k = 0; k < SN; ++k) a = fmaf(S[i * SN + k], F[k * SN + j], a);
                SF[i * SN + j] = a;
            }
#pragma unroll
        for (int e = 0; e < SNN; ++e) S[e] += SF[e];
        float4* o = reinterpret_cast<float4*>(S_out + row);
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
    }
}

// Whether a problem runs on k_small_scan (its chunk is the whole sequence).
bool small_scan_ok(const KParams& p, bool readout)
{
    return p.n == SN && !readout && p.K == 1 &&
           (p.src != SRC_EMBEDDING || p.mode == MRU_MODE_RESHAPE || p.mode == MRU_MODE_DETNORM ||
            p.mode == MRU_MODE_LDU);
}

template <int N>
cudaError_t scan_n(const KParams& p, const void* src, const float* S0, const float* u, int64_t snap_every,
                   float* S_out, float* o_out, float* snaps, char* ws, const Workspace& W, cudaStream_t s,
                   int* launches)
{
    constexpr int NN = N * N;
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + W.status);
    float* totals = reinterpret_cast<float*>(ws + W.totals);
    double* local = reinterpret_cast<double*>(ws + W.local);
    double* gcarry = reinterpret_cast<double*>(ws + W.gcarry);
    float* carry = reinterpret_cast<float*>(ws + W.carry);
    const int64_t BH = p.B * p.H;
    const int64_t chains = BH * p.K;
    if (chains == 0) return cudaSuccess;
    cudaError_t e;

    // the chunk kernel: one CTA per chain (one warp per chain measured no
    // faster here: 0.87x to 1.21x of the CTA time across modes at n = 16)
    using Grp = CtaGroup;
    constexpr int GPB = kThreads / Grp::kSize;
    const int gfl = 4 * NN + 4 * N + 8 + N * p.rq;
    const size_t sm_chunk = sizeof(float) * gfl * GPB;
    const unsigned grid_chunk = (unsigned)((chains + GPB - 1) / GPB);
    const size_t sm_d = sizeof(double) * 2 * N * CarryMul<N>::SP;
    const size_t sm_fix = sizeof(float) * (2 * NN + N * p.rq);
    if ((e = set_smem(k_chunk_prefix<N, Grp>, sm_chunk)) != cudaSuccess) return e;
    if ((e = set_smem(k_carry_local<N>, sm_d)) != cudaSuccess) return e;
    if ((e = set_smem(k_carry_groups<N>, sm_d)) != cudaSuccess) return e;
    if ((e = set_smem(k_carry_final<N>, sm_d)) != cudaSuccess) return e;
    if ((e = set_smem(k_fixup<N>, sm_fix)) != cudaSuccess) return e;
    profile_mark(0, 0, s);
    if (N == SN && small_scan_ok(p, o_out != nullptr)) {
        k_small_scan<<<(unsigned)BH, kThreads, 0, s>>>(p, src, S_out, S0, status);
        profile_mark(0, 1, s);
        if (launches) *launches = 1;
        return cudaGetLastError();
    }
    if (p.K == 1) {
        // one chunk per sequence: the chunk kernel starts from S0 and its
        // outputs are final (the decode / short-segment latency path)
        k_chunk_prefix<N, Grp><<<grid_chunk, kThreads, sm_chunk, s>>>(p, src, u, snap_every, S_out, o_out,
                                                                       snaps, totals, status, S0, 1, gfl);
        profile_mark(0, 1, s);
        if (launches) *launches = 1;
        return cudaGetLastError();
    }
    // n = 64 on the tensor cores: the readout form, or every state as a
    // snapshot at every token (no query columns)
    const bool fast64 = N == 64 && n64::supports(p, o_out != nullptr);
    KParams p64 = p;
    if (fast64 && o_out == nullptr) p64.rq = 0;
    if (fast64) {
        if ((e = n64::launch_chunk_readout(p64, reinterpret_cast<const float*>(src), u, o_out ? snap_every : 1,
                                           o_out, o_out ? snaps : S_out, totals, status, s)) != cudaSuccess)
            return e;
    } else {
        k_chunk_prefix<N, Grp><<<grid_chunk, kThreads, sm_chunk, s>>>(p, src, u, snap_every, S_out, o_out,
                                                                       snaps, totals, status, nullptr, 0, gfl);
    }
    profile_mark(0, 1, s);
    profile_mark(1, 0, s);
    k_carry_local<N><<<(unsigned)(BH * p.NG), kThreads, sm_d, s>>>(p, totals, local);
    profile_mark(1, 1, s);
    profile_mark(2, 0, s);
    k_carry_groups<N><<<(unsigned)BH, kThreads, sm_d, s>>>(p, S0, local, gcarry);
    profile_mark(2, 1, s);
    profile_mark(3, 0, s);
    k_carry_final<N><<<(unsigned)chains, kThreads, sm_d, s>>>(p, local, gcarry, carry);
    profile_mark(3, 1, s);
    profile_mark(4, 0, s);
    if (fast64) {
        if ((e = n64::launch_fixup_readout(p64, carry, u, o_out ? snap_every : 1, o_out, o_out ? snaps : S_out, s)) !=
            cudaSuccess)
            return e;
    } else {
        k_fixup<N><<<(unsigned)chains, kThreads, sm_fix, s>>>(p, carry, u, snap_every, S_out, o_out, snaps);
    }
    profile_mark(4, 1, s);
    if (launches) *launches = 5;
    return cudaGetLastError();
}

cudaError_t scan_fast16(const KParams& p, const void* src, const float* S0, float* S_out, char* ws,
                        const Workspace& W, cudaStream_t s, int* launches)
{
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + W.status);
    float* totals = reinterpret_cast<float*>(ws + W.totals);
    const float* x = reinterpret_cast<const float*>(src);
    if (p.B * p.H * p.K == 0) return cudaSuccess;
    cudaError_t e;
    if (p.K == 1) {
        // one chunk per sequence: the apply pass alone, from S0
        profile_mark(0, 0, s);
        if ((e = n16::launch_apply(p, x, W.c16, ws, S_out, status, S0, true, false, s)) != cudaSuccess) return e;
        profile_mark(0, 1, s);
        if (launches) *launches = 1;
        return cudaGetLastError();
    }
    if (W.fused) {
        profile_mark(0, 0, s);
        if ((e = n16::launch_fused(p, W.f16, ws, x, S0, S_out, status, s)) != cudaSuccess) return e;
        profile_mark(0, 1, s);
        if (launches) *launches = 1;
        return cudaGetLastError();
    }
    profile_mark(0, 0, s);
    float* fbuf = W.fstore ? reinterpret_cast<float*>(ws + W.fbuf) : nullptr;
    if ((e = n16::launch_reduce(p, x, totals, W.c16, ws, status, fbuf, s)) != cudaSuccess) return e;
    profile_mark(0, 1, s);
    profile_mark(1, 0, s);
    if ((e = n16::launch_carry(p, totals, W.c16, ws, S0, s)) != cudaSuccess) return e;
    profile_mark(1, 1, s);
    profile_mark(2, 0, s);
    if ((e = n16::launch_apply(p, fbuf ? fbuf : x, W.c16, ws, S_out, status, nullptr, false, fbuf != nullptr, s)) !=
        cudaSuccess)
        return e;
    profile_mark(2, 1, s);
    if (launches) *launches = 3;
    return cudaGetLastError();
}

cudaError_t scan_fast32(const KParams& p, const void* src, const float* S0, float* S_out, char* ws,
                        const Workspace& W, cudaStream_t s, int* launches)
{
    float* totals = reinterpret_cast<float*>(ws + W.totals);
    if (p.B * p.H * p.K == 0) return cudaSuccess;
    cudaError_t e;
    int slot = 0;
    if (p.K == 1) {
        profile_mark(0, 0, s);
        if ((e = n32::launch_apply(p, src, W.plan, ws, S_out, S0, true, s)) != cudaSuccess) return e;
        profile_mark(0, 1, s);
        if (launches) *launches = 1;
        return cudaGetLastError();
    }
    profile_mark(slot, 0, s);
    if ((e = n32::launch_reduce(p, src, totals, s)) != cudaSuccess) return e;
    profile_mark(slot++, 1, s);
    if ((e = carry::run_n32(W.plan, totals, S0, ws, s, slot)) != cudaSuccess) return e;
    profile_mark(slot, 0, s);
    if ((e = n32::launch_apply(p, src, W.plan, ws, S_out, nullptr, false, s)) != cudaSuccess) return e;
    profile_mark(slot++, 1, s);
    if (launches) *launches = slot;
    return cudaGetLastError();
}

}  // namespace

int32_t effective_math(const KParams& p, bool readout)
{
    if (n16::supports(p, readout)) return MRU_MATH_TF32X3;
    if (n32::supports(p, readout)) return MRU_MATH_BF16X3;
    if (n64::supports(p, readout)) return MRU_MATH_TF32;
    return MRU_MATH_FP32;
}

const char* kernel_name(const KParams& p, bool readout, int i)
{
    static const char* generic[] = {"k_chunk_prefix", "k_carry_local", "k_carry_groups", "k_carry_final",
                                    "k_fixup"};
    if (i < 0 || i >= (p.K == 1 ? 1 : 5)) return "";
    if (i == 0 && small_scan_ok(p, readout)) return "k_small_scan";
    if (i == 0 && n64::supports(p, readout)) return n64::use_tcgen05() ? "k64_chunk_readout_tc" : "k64_chunk_readout";
    if (i == 4 && n64::supports(p, readout)) return "k64_fixup";
    return generic[i];
}

cudaError_t launch_build_states(const KParams& p, const void* x, float* X_out, int store_minus_identity,
                                void* ws_base, const Workspace& W, cudaStream_t s)
{
    uint32_t* status = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws_base) + W.status);
    switch (p.n) {
        case 4: return build_states_n<4>(p, x, X_out, store_minus_identity, status, s);
        case 8: return build_states_n<8>(p, x, X_out, store_minus_identity, status, s);
        case 16: return build_states_n<16>(p, x, X_out, store_minus_identity, status, s);
        case 32: return build_states_n<32>(p, x, X_out, store_minus_identity, status, s);
        case 64: return build_states_n<64>(p, x, X_out, store_minus_identity, status, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan(const KParams& p, const void* src, const float* S0, const float* u,
                        int64_t snap_every, float* S_out, float* o_out, float* snaps,
                        void* ws_base, const Workspace& W, cudaStream_t s, int* launches)
{
    char* ws = reinterpret_cast<char*>(ws_base);
    if (W.fast && W.fast_n == 32) return scan_fast32(p, src, S0, S_out, ws, W, s, launches);
    if (W.fast) return scan_fast16(p, src, S0, S_out, ws, W, s, launches);
    switch (p.n) {
        case 4: return scan_n<4>(p, src, S0, u, snap_every, S_out, o_out, snaps, ws, W, s, launches);
        case 8: return scan_n<8>(p, src, S0, u, snap_every, S_out, o_out, snaps, ws, W, s, launches);
        case 16: return scan_n<16>(p, src, S0, u, snap_every, S_out, o_out, snaps, ws, W, s, launches);
        case 32: return scan_n<32>(p, src, S0, u, snap_every, S_out, o_out, snaps, ws, W, s, launches);
        case 64: return scan_n<64>(p, src, S0, u, snap_every, S_out, o_out, snaps, ws, W, s, launches);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_backward(const KParams& p, const void* x, const float* S0, const float* S_fwd, const float* dS,
                            float* dx, float* dS0, void* ws_base, const BwdWorkspace& W, cudaStream_t s)
{
    char* ws = reinterpret_cast<char*>(ws_base);
    switch (p.n) {
        case 4: return backward_n<4>(p, x, S0, S_fwd, dS, dx, dS0, ws, W, s);
        case 8: return backward_n<8>(p, x, S0, S_fwd, dS, dx, dS0, ws, W, s);
        case 16: return backward_n<16>(p, x, S0, S_fwd, dS, dx, dS0, ws, W, s);
        case 32: return backward_n<32>(p, x, S0, S_fwd, dS, dx, dS0, ws, W, s);
        case 64: return backward_n<64>(p, x, S0, S_fwd, dS, dx, dS0, ws, W, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace mru
