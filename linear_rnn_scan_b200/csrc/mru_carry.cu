// mru_carry.cu -- multi-level fp64 scan of chunk totals for the n = 32
// kernels (one CTA of 8 warps per group of G matrices; every 32 x 32 product
// on the fp64 tensor cores, mma.sync m8n8k4, operands in shared memory).
//
// Level 1 sees the chunk totals T_k = I + Q_k (fp32 Q_k from the chunk
// kernel).  Each level cuts its sequence of matrices into groups of G and
// forms, per group, the inclusive local prefixes R_j = prefix - I (fp64, split
// form, R_j = R_{j-1} + (T_j + R_{j-1} T_j)) and the group total.  The group
// totals are the next level's input; the top level (at most G matrices per
// sequence) is scanned from S0 into exclusive carries E_top.  Going back down,
// E_l[i] = E_{l+1}[i / G] (I + R_l[i - 1]) (or E_{l+1}[i / G] for the first
// of a group).  The level-1 carries are formed by the apply kernel itself.
//
// Local prefixes of level 1 are stored in fp32 (they span at most G chunks
// and are used once, by the apply pass); every prefix that feeds a longer
// chain stays fp64.
#include <string.h>

#include "mru_internal.cuh"

namespace mru {
namespace carry {
namespace {

constexpr int N = 32;
constexpr int NN = N * N;
constexpr int SN = 36;               // padded shared-memory row stride (doubles)
constexpr int SNN = N * SN;          // one staged matrix
constexpr int CT = 256;              // 8 warps

// D += A B, m8n8k4, fp64 throughout.
__device__ __forceinline__ void mma_f64(double (&d)[2], double a, double b)
{
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
                 : "+d"(d[0]), "+d"(d[1])
                 : "d"(a), "d"(b));
}

// The CTA's product of two 32 x 32 fp64 matrices in shared memory (row
// stride SN; with SN = 36 the fragment reads of a half-warp hit 16 distinct
// 8-byte banks).  Warp w computes rows 8 (w / 2) ... + 7 and columns
// 16 (w % 2) ... + 15; thread output r (0..3) is element out_pos(r).
struct CtaMul {
    static constexpr int PER = 4;
    __device__ static void pos(int r, int& row, int& col)
    {
        const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
        row = 8 * (w >> 1) + (lane >> 2);
        col = 16 * (w & 1) + 8 * (r >> 1) + 2 * (lane & 3) + (r & 1);
    }
    __device__ static void mul(const double* A, const double* B, double (&acc)[PER])
    {
        const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
        const double* Ar = A + (8 * (w >> 1) + g) * SN + t;
        const double* Bc = B + t * SN + 16 * (w & 1) + g;
        double d[2][2][2];                   // column tile, k half, element
#pragma unroll
        for (int i = 0; i < 8; ++i) (&d[0][0][0])[i] = 0.0;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const double a = Ar[4 * kk];
#pragma unroll
            for (int j = 0; j < 2; ++j) mma_f64(d[j][kk >> 2], a, Bc[4 * kk * SN + 8 * j]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) acc[2 * j + h] = d[j][0][h] + d[j][1][h];
    }
};

// Copies `count` row-major N x N matrices (fp32 when in32, else fp64) to
// shared memory as fp64 with padded rows, every load in flight at once.
__device__ __forceinline__ void stage(double* dst, const void* src, int64_t base, int64_t nvals, int in32)
{
    if (in32) {
        const float4* s4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + base);
        for (int64_t e = threadIdx.x; e < nvals / 4; e += CT) {
            const float4 v = s4[e];
            const int64_t m = (4 * e) / NN;
            const int idx = (int)((4 * e) % NN), row = idx / N, col = idx % N;
            double* d = dst + m * SNN + row * SN + col;
            d[0] = v.x;
            d[1] = v.y;
            d[2] = v.z;
            d[3] = v.w;
        }
    } else {
        const double2* s2 = reinterpret_cast<const double2*>(reinterpret_cast<const double*>(src) + base);
        for (int64_t e = threadIdx.x; e < nvals / 2; e += CT) {
            const double2 v = s2[e];
            const int64_t m = (2 * e) / NN;
            const int idx = (int)((2 * e) % NN), row = idx / N, col = idx % N;
            double* d = dst + m * SNN + row * SN + col;
            d[0] = v.x;
            d[1] = v.y;
        }
    }
}

// Inclusive local prefixes of one level.  Input: per sequence `cnt` matrices
// (fp32 split form when in32, else fp64 split form), laid out
// [seq][cnt][N][N].  Output: R (fp32 when out32, else fp64) [seq][cnt], and
// group totals Tot (fp64) [seq][ceil(cnt / G)].  One CTA per (seq, group);
// the group's inputs are staged in shared memory first.
__global__ void __launch_bounds__(CT)
k_level(int64_t nseq, int64_t cnt, int G, const void* in, int in32, void* R, int out32, double* Tot)
{
    extern __shared__ double dyn[];
    double* sR = dyn;
    double* sIn = sR + SNN;
    const int64_t ngroups = (cnt + G - 1) / G;
    const int64_t seq = blockIdx.x / ngroups, g = blockIdx.x % ngroups;
    const int64_t j0 = g * G, j1 = (j0 + G < cnt) ? j0 + G : cnt;
    stage(sIn, in, (seq * cnt + j0) * NN, (j1 - j0) * NN, in32);
    for (int e = threadIdx.x; e < SNN; e += CT) sR[e] = 0.0;
    __syncthreads();
    for (int64_t j = j0; j < j1; ++j) {
        const double* sT = sIn + (j - j0) * SNN;
        const int64_t base = (seq * cnt + j) * NN;
        double acc[CtaMul::PER];
        CtaMul::mul(sR, sT, acc);
        __syncthreads();
#pragma unroll
        for (int r = 0; r < CtaMul::PER; ++r) {
            int row, col;
            CtaMul::pos(r, row, col);
            const double v = sR[row * SN + col] + (sT[row * SN + col] + acc[r]);
            sR[row * SN + col] = v;
            if (out32) reinterpret_cast<float*>(R)[base + row * N + col] = (float)v;
            else reinterpret_cast<double*>(R)[base + row * N + col] = v;
        }
        __syncthreads();
    }
    double* tot = Tot + (seq * ngroups + g) * NN;
    for (int e = threadIdx.x; e < NN; e += CT) tot[e] = sR[(e / N) * SN + e % N];
}

// Top level: exclusive carries of at most G group totals per sequence,
// starting from S0 (or I).  E[seq][i] = S0 prod_{m < i} (I + Tot_m).
__global__ void __launch_bounds__(CT)
k_top(int64_t nseq, int64_t cnt, int G, const double* Tot, const float* S0, double* E)
{
    extern __shared__ double dyn[];
    double* sG = dyn;
    double* sIn = sG + SNN;
    const int64_t seq = blockIdx.x;
    (void)G;
    stage(sIn, Tot, seq * cnt * NN, cnt * NN, 0);
    for (int e = threadIdx.x; e < NN; e += CT)
        sG[(e / N) * SN + e % N] = S0 ? (double)S0[seq * NN + e] : ((e / N) == (e % N) ? 1.0 : 0.0);
    __syncthreads();
    for (int64_t i = 0; i < cnt; ++i) {
        const double* sT = sIn + i * SNN;
        const int64_t base = (seq * cnt + i) * NN;
        for (int e = threadIdx.x; e < NN; e += CT) E[base + e] = sG[(e / N) * SN + e % N];
        double acc[CtaMul::PER];
        CtaMul::mul(sG, sT, acc);
        __syncthreads();
#pragma unroll
        for (int r = 0; r < CtaMul::PER; ++r) {
            int row, col;
            CtaMul::pos(r, row, col);
            sG[row * SN + col] += acc[r];
        }
        __syncthreads();
    }
}

// Going down one level: E_l[i] = E_{l+1}[i / G] (I + R_l[i - 1]), with R_l
// fp64.  One CTA per matrix.
__global__ void __launch_bounds__(CT)
k_down(int64_t nseq, int64_t cnt, int G, const double* Eup, const double* R, double* E)
{
    extern __shared__ double dyn[];
    double* sG = dyn;
    double* sT = sG + SNN;
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
        sG[(e / N) * SN + e % N] = up[e];
        sT[(e / N) * SN + e % N] = rp[e];
    }
    __syncthreads();
    double acc[CtaMul::PER];
    CtaMul::mul(sG, sT, acc);
#pragma unroll
    for (int r = 0; r < CtaMul::PER; ++r) {
        int row, col;
        CtaMul::pos(r, row, col);
        out[row * N + col] = sG[row * SN + col] + acc[r];
    }
}

cudaError_t run(const Plan& pl, const float* totals, const float* S0, char* ws, cudaStream_t s, int& slot)
{
    const int64_t nseq = pl.nseq;
    // level 1: chunk totals (fp32) -> R1 (fp32), Tot1 (fp64)
    int64_t cnt = pl.cnt[0];
    const void* in = totals;
    int in32 = 1;
    const size_t sm = sizeof(double) * (size_t)(pl.G + 1) * SNN;
    cudaError_t e = cudaFuncSetAttribute(k_level, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_top, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    for (int l = 0; l < pl.levels; ++l) {
        const int64_t ng = (cnt + pl.G - 1) / pl.G;
        profile_mark(slot, 0, s);
        k_level<<<(unsigned)(nseq * ng), CT, sm, s>>>(nseq, cnt, pl.G, in, in32, ws + pl.R[l], l == 0 ? 1 : 0,
                                                      reinterpret_cast<double*>(ws + pl.Tot[l]));
        profile_mark(slot++, 1, s);
        in = ws + pl.Tot[l];
        in32 = 0;
        cnt = ng;
    }
    // top
    profile_mark(slot, 0, s);
    k_top<<<(unsigned)nseq, CT, sm, s>>>(nseq, cnt, pl.G, reinterpret_cast<const double*>(in), S0,
                                         reinterpret_cast<double*>(ws + pl.E[pl.levels]));
    profile_mark(slot++, 1, s);
    // down to level 2's carries (level-1 carries are formed by the apply pass)
    const size_t sm2 = sizeof(double) * 2 * SNN;
    for (int l = pl.levels - 1; l >= 1; --l) {
        const int64_t c = pl.cnt[l];
        profile_mark(slot, 0, s);
        k_down<<<(unsigned)(nseq * c), CT, sm2, s>>>(nseq, c, pl.G,
                                                     reinterpret_cast<const double*>(ws + pl.E[l + 1]),
                                                     reinterpret_cast<const double*>(ws + pl.R[l]),
                                                     reinterpret_cast<double*>(ws + pl.E[l]));
        profile_mark(slot++, 1, s);
    }
    return cudaGetLastError();
}}  // namespace

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
    return run(pl, totals, S0, ws, s, slot);
}

}  // namespace carry
}  // namespace mru
