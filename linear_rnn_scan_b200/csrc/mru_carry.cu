// mru_carry.cu -- multi-level fp64 scan of chunk totals for the n = 32
// kernels (one CTA per group of G matrices, every thread one output element
// of each small product).
//
// Level 1 sees the chunk totals T_k = I + Q_k (fp32 Q_k from the chunk
// kernel).  Each level cuts its sequence of matrices into groups of G and
// forms, per group, the inclusive local prefixes R_j = prefix - I (fp64, split
// form, R_j = R_{j-1} + (T_j + R_{j-1} T_j)) and the group total.  The group
// totals are the next level's input; the top level (at most G matrices per
// sequence) is scanned from S0 into exclusive carries E_top.  Going back down,
// E_l[i] = E_{l+1}[i / G] (I + R_l[i - 1]) (or E_{l+1}[i / G] for the first
// of a group).  The level-1 carries are formed by the fix-up kernel itself.
//
// Local prefixes of level 1 are stored in fp32 (they span at most G chunks
// and are used once, by the fix-up); every prefix that feeds a longer chain
// stays fp64.
#include <string.h>

#include "mru_internal.cuh"

namespace mru {
namespace carry {
namespace {

constexpr int CT = 256;              // threads per CTA: one CTA per group / sequence / matrix

// Cooperative fp64 product of two N x N matrices in shared memory: thread t
// computes outputs (i, j) for e = t, t + CT, ... (i = e / N, j = e % N); the
// whole CTA calls it.  PER = N*N / CT outputs per thread.
template <int N>
struct CtaGemm {
    static constexpr int PER = (N * N + CT - 1) / CT;
    __device__ static void mul(const double* A, const double* B, double (&acc)[PER])
    {
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int e = threadIdx.x + r * CT;
            const int i = e / N, j = e % N;
            double a = 0.0;
#pragma unroll 8
            for (int k = 0; k < N; ++k) a = fma(A[i * N + k], B[k * N + j], a);
            acc[r] = a;
        }
    }
};

// Copies `count` N x N matrices (fp32 when in32, else fp64) to shared memory
// as fp64, every load in flight at once.
__device__ __forceinline__ void stage(double* dst, const void* src, int64_t base, int64_t nvals, int in32)
{
    if (in32) {
        const float4* s4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + base);
        for (int64_t e = threadIdx.x; e < nvals / 4; e += CT) {
            const float4 v = s4[e];
            dst[4 * e + 0] = v.x;
            dst[4 * e + 1] = v.y;
            dst[4 * e + 2] = v.z;
            dst[4 * e + 3] = v.w;
        }
    } else {
        const double2* s2 = reinterpret_cast<const double2*>(reinterpret_cast<const double*>(src) + base);
        for (int64_t e = threadIdx.x; e < nvals / 2; e += CT) {
            const double2 v = s2[e];
            dst[2 * e + 0] = v.x;
            dst[2 * e + 1] = v.y;
        }
    }
}

// Inclusive local prefixes of one level.  Input: per sequence `cnt` matrices
// (fp32 split form when in32, else fp64 split form), laid out
// [seq][cnt][N][N].  Output: R (fp32 when out32, else fp64) [seq][cnt], and
// group totals Tot (fp64) [seq][ceil(cnt / G)].  One CTA per (seq, group);
// the group's inputs are staged in shared memory first.
template <int N>
__global__ void __launch_bounds__(CT)
k_level(int64_t nseq, int64_t cnt, int G, const void* in, int in32, void* R, int out32, double* Tot)
{
    constexpr int NN = N * N;
    using CG = CtaGemm<N>;
    extern __shared__ double dyn[];
    double* sR = dyn;
    double* sIn = sR + NN;
    const int64_t ngroups = (cnt + G - 1) / G;
    const int64_t seq = blockIdx.x / ngroups, g = blockIdx.x % ngroups;
    const int64_t j0 = g * G, j1 = (j0 + G < cnt) ? j0 + G : cnt;
    stage(sIn, in, (seq * cnt + j0) * NN, (j1 - j0) * NN, in32);
    for (int e = threadIdx.x; e < NN; e += CT) sR[e] = 0.0;
    __syncthreads();
    for (int64_t j = j0; j < j1; ++j) {
        const double* sT = sIn + (j - j0) * NN;
        const int64_t base = (seq * cnt + j) * NN;
        double acc[CG::PER];
        CG::mul(sR, sT, acc);
        __syncthreads();
#pragma unroll
        for (int r = 0; r < CG::PER; ++r) {
            const int e = threadIdx.x + r * CT;
            const double v = sR[e] + (sT[e] + acc[r]);
            sR[e] = v;
            if (out32) reinterpret_cast<float*>(R)[base + e] = (float)v;
            else reinterpret_cast<double*>(R)[base + e] = v;
        }
        __syncthreads();
    }
    double* tot = Tot + (seq * ngroups + g) * NN;
    for (int e = threadIdx.x; e < NN; e += CT) tot[e] = sR[e];
}

// Top level: exclusive carries of at most G group totals per sequence,
// starting from S0 (or I).  E[seq][i] = S0 prod_{m < i} (I + Tot_m).
template <int N>
__global__ void __launch_bounds__(CT)
k_top(int64_t nseq, int64_t cnt, int G, const double* Tot, const float* S0, double* E)
{
    constexpr int NN = N * N;
    using CG = CtaGemm<N>;
    extern __shared__ double dyn[];
    double* sG = dyn;
    double* sIn = sG + NN;
    const int64_t seq = blockIdx.x;
    (void)G;
    stage(sIn, Tot, seq * cnt * NN, cnt * NN, 0);
    for (int e = threadIdx.x; e < NN; e += CT)
        sG[e] = S0 ? (double)S0[seq * NN + e] : ((e / N) == (e % N) ? 1.0 : 0.0);
    __syncthreads();
    for (int64_t i = 0; i < cnt; ++i) {
        const double* sT = sIn + i * NN;
        const int64_t base = (seq * cnt + i) * NN;
        for (int e = threadIdx.x; e < NN; e += CT) E[base + e] = sG[e];
        double acc[CG::PER];
        CG::mul(sG, sT, acc);
        __syncthreads();
#pragma unroll
        for (int r = 0; r < CG::PER; ++r) {
            const int e = threadIdx.x + r * CT;
            sG[e] = sG[e] + acc[r];
        }
        __syncthreads();
    }
}

// Going down one level: E_l[i] = E_{l+1}[i / G] (I + R_l[i - 1]), with R_l
// fp64.  One CTA per matrix.
template <int N>
__global__ void __launch_bounds__(CT)
k_down(int64_t nseq, int64_t cnt, int G, const double* Eup, const double* R, double* E)
{
    constexpr int NN = N * N;
    using CG = CtaGemm<N>;
    __shared__ double sG[NN];
    __shared__ double sT[NN];
    const int64_t item = blockIdx.x;
    const int64_t seq = item / cnt, i = item % cnt;
    const int64_t nup = (cnt + G - 1) / G;
    const double* up = Eup + (seq * nup + i / G) * NN;
    double* out = E + item * NN;
    if (i % G == 0) {
        for (int e = threadIdx.x; e < NN; e += CT) out[e] = up[e];
        return;
    }
    const double* rp = R + (item - 1) * NN;
    for (int e = threadIdx.x; e < NN; e += CT) {
        sG[e] = up[e];
        sT[e] = rp[e];
    }
    __syncthreads();
    double acc[CG::PER];
    CG::mul(sG, sT, acc);
#pragma unroll
    for (int r = 0; r < CG::PER; ++r) {
        const int e = threadIdx.x + r * CT;
        out[e] = sG[e] + acc[r];
    }
}

template <int N>
cudaError_t run(const Plan& pl, const float* totals, const float* S0, char* ws, cudaStream_t s, int& slot)
{
    constexpr int NN = N * N;
    const int64_t nseq = pl.nseq;
    // level 1: chunk totals (fp32) -> R1 (fp32), Tot1 (fp64)
    int64_t cnt = pl.cnt[0];
    const void* in = totals;
    int in32 = 1;
    const size_t sm = sizeof(double) * (size_t)(pl.G + 1) * NN;
    cudaError_t e = cudaFuncSetAttribute(k_level<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_top<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    for (int l = 0; l < pl.levels; ++l) {
        const int64_t ng = (cnt + pl.G - 1) / pl.G;
        profile_mark(slot, 0, s);
        k_level<N><<<(unsigned)(nseq * ng), CT, sm, s>>>(nseq, cnt, pl.G, in, in32, ws + pl.R[l], l == 0 ? 1 : 0,
                                                         reinterpret_cast<double*>(ws + pl.Tot[l]));
        profile_mark(slot++, 1, s);
        in = ws + pl.Tot[l];
        in32 = 0;
        cnt = ng;
    }
    // top
    profile_mark(slot, 0, s);
    k_top<N><<<(unsigned)nseq, CT, sm, s>>>(nseq, cnt, pl.G, reinterpret_cast<const double*>(in), S0,
                                            reinterpret_cast<double*>(ws + pl.E[pl.levels]));
    profile_mark(slot++, 1, s);
    // down to level 2's carries (level-1 carries are formed by the apply pass)
    for (int l = pl.levels - 1; l >= 1; --l) {
        const int64_t c = pl.cnt[l];
        profile_mark(slot, 0, s);
        k_down<N><<<(unsigned)(nseq * c), CT, 0, s>>>(nseq, c, pl.G,
                                                      reinterpret_cast<const double*>(ws + pl.E[l + 1]),
                                                      reinterpret_cast<const double*>(ws + pl.R[l]),
                                                      reinterpret_cast<double*>(ws + pl.E[l]));
        profile_mark(slot++, 1, s);
    }
    return cudaGetLastError();
}

}  // namespace

// Plan the levels for `nseq` sequences of `K` chunk totals each, with the
// workspace laid out from byte offset `off`.  Level l has cnt[l] matrices per
// sequence; R[l] (fp32 for l == 0, fp64 above) and Tot[l] (fp64) hold its
// local prefixes and group totals; E[l] holds the exclusive carries of level l
// (E[0] is not stored: the fix-up forms it).
Plan plan(int64_t nseq, int64_t K, int nn, size_t off)
{
    Plan pl;
    memset(&pl, 0, sizeof pl);
    pl.nseq = nseq;
    pl.G = nn <= 256 ? 16 : 8;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) / 256 * 256;
        return o;
    };
    int64_t cnt = K;
    int l = 0;
    pl.cnt[0] = K;
    // levels until the top has at most G matrices per sequence (at least one
    // level so that the fix-up always finds R_1 and E_1's parent)
    do {
        const int64_t ng = (cnt + pl.G - 1) / pl.G;
        pl.R[l] = take((size_t)nseq * cnt * nn * (l == 0 ? sizeof(float) : sizeof(double)));
        pl.Tot[l] = take((size_t)nseq * ng * nn * sizeof(double));
        cnt = ng;
        pl.cnt[++l] = cnt;
    } while (cnt > pl.G && l < kMaxLevels - 1);
    pl.levels = l;
    for (int i = 1; i <= l; ++i) pl.E[i] = take((size_t)nseq * pl.cnt[i] * nn * sizeof(double));
    pl.end = off;
    return pl;
}

int launches(const Plan& pl) { return pl.levels + 1 + (pl.levels - 1); }

cudaError_t run_n32(const Plan& pl, const float* totals, const float* S0, char* ws, cudaStream_t s, int& slot)
{
    return run<32>(pl, totals, S0, ws, s, slot);
}

}  // namespace carry
}  // namespace mru
