// mru_n16.cu -- n = 16 scan kernels on the tensor cores (fp32 embeddings,
// reshape and determinant-corrected modes).
//
// Same three phases and numerics as the generic path (identity split,
// product term accumulated apart, fp64 per-token scalars, fp64 chunk-total
// scan), mapped onto the B200 this way:
//
//  * chunk kernel  one warp per chain (b, h, chunk of 8 tokens), 8 chains per
//                  CTA.  Phase 1: the CTA copies its 64 token-head slices to
//                  shared memory (cp.async, rows padded to 20 words) and runs
//                  64 LU factorisations at once, 4 lanes per token (each lane
//                  owns rows r, r+4, r+8, r+12 in registers; the pivot row is
//                  broadcast by shuffles inside the 4-lane group).  Phase 2:
//                  each warp runs its chain Q_t = Q_{t-1} + (F_t + Q_{t-1} F_t)
//                  with mma.sync m16n8k8 tf32 in split precision (hi + lo
//                  operands, three products), the state staying in the
//                  accumulator registers from step to step: the contraction
//                  index of the next product is permuted so that the
//                  accumulator fragment of column tile j is exactly the A
//                  fragment of k-tile j.
//  * fix-up kernel one warp per chain: S_t = C + C Q_t with the carry C as the
//                  split A operand (loaded once) and Q_t streamed in.
//
// Split-tf32 ("3xTF32", after Ootomo and Yokota, 2022): x = hi + lo with hi
// the top 19 bits of x (sign, exponent, 10 mantissa bits) and lo = x - hi
// exact in fp32; a b ~ a_hi b_hi + a_hi b_lo + a_lo b_hi, the small terms
// first.
#include "mru_internal.cuh"

namespace mru {
namespace n16 {
namespace {

constexpr int N = 16;
constexpr int NN = N * N;
constexpr int ROWW = 20;            // padded shared-memory row stride, in words
constexpr int SLICE = N * ROWW;     // one token-head slice in shared memory
constexpr int CT = 8;               // tokens per chunk
constexpr int WARPS = 8;            // chains per CTA
constexpr int THREADS = 32 * WARPS;

struct Smem {
    float x[WARPS][CT][SLICE];      // 81,920 bytes
    float c[WARPS][CT][2];          // c_t and c_t - 1
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::); }

__device__ __forceinline__ void split_tf32(float v, uint32_t& hi, uint32_t& lo)
{
    const uint32_t h = __float_as_uint(v) & 0xffffe000u;
    hi = h;
    lo = __float_as_uint(v - __uint_as_float(h));
}

// D += A B, m16n8k8, tf32 operands, fp32 accumulate.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc += A B in split precision for one (k-tile, n-tile) pair.
__device__ __forceinline__ void mma_3xtf32(float (&acc)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                           const uint32_t (&bh)[2], const uint32_t (&bl)[2])
{
    mma_tf32(acc, al, bh);
    mma_tf32(acc, ah, bl);
    mma_tf32(acc, ah, bh);
}

// log|det(W)| of one 16 x 16 matrix held by a group of 4 lanes (lane r of
// the group owns rows r, r+4, r+8, r+12 in e[0..3][0..15]).  near_identity:
// W = I + e, eliminated on e alone without pivoting; returns false (and
// nothing useful) when a pivot |1 + delta_k| < 0.5.  Otherwise W = e with
// partial pivoting.  The determinant magnitude is accumulated in fp64.
__device__ __forceinline__ bool group_logabsdet(float (&e)[4][N], int r, bool near_identity, double& logabs,
                                                bool& singular)
{
    const unsigned full = 0xffffffffu;
    double prod = 1.0;
    double lsum = 0.0;
    bool ok = true;
    singular = false;
#pragma unroll
    for (int k = 0; k < N; ++k) {
        const int kr = k >> 2, owner = k & 3;
        if (!near_identity) {
            // partial pivoting: largest |W[i][k]| over rows i >= k of the group
            float best = -1.0f;
            int bi = k;
#pragma unroll
            for (int lr = 0; lr < 4; ++lr) {
                const int i = 4 * lr + r;
                const float a = fabsf(e[lr][k]);
                if (i >= k && a > best) { best = a; bi = i; }
            }
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                const float ob = __shfl_xor_sync(full, best, o, 4);
                const int oi = __shfl_xor_sync(full, bi, o, 4);
                if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            if (!(best > 0.0f)) singular = true;
            {
                // swap rows k and bi (row i lives in lane i & 3, slot i >> 2);
                // executed unconditionally (a no-op when bi == k) so that the
                // shuffles stay converged across the warp
                const int pr = bi >> 2, powner = bi & 3;
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    float vk = 0.0f, vp = 0.0f;
#pragma unroll
                    for (int lr = 0; lr < 4; ++lr) {
                        if (lr == kr) vk = e[lr][j];
                        if (lr == pr) vp = e[lr][j];
                    }
                    const float rowk = __shfl_sync(full, vk, owner, 4);
                    const float rowp = __shfl_sync(full, vp, powner, 4);
#pragma unroll
                    for (int lr = 0; lr < 4; ++lr) {
                        if (lr == kr && r == owner) e[lr][j] = rowp;
                        if (lr == pr && r == powner) e[lr][j] = rowk;
                    }
                }
            }
        }
        // broadcast pivot row k from its owner lane
        float prow[N];
#pragma unroll
        for (int j = 0; j < N; ++j) {
            if (j >= k) {
                float v = 0.0f;
#pragma unroll
                for (int lr = 0; lr < 4; ++lr)
                    if (lr == kr) v = e[lr][j];
                prow[j] = __shfl_sync(full, v, owner, 4);
            }
        }
        float pk;
        if (near_identity) {
            const float d = prow[k];
            pk = 1.0f + d;
            if (!(fabsf(pk) >= 0.5f)) ok = false;
            prod *= 1.0 + (double)d;
        } else {
            pk = prow[k];
            lsum += log(fabs((double)pk));
        }
        const float rk = (pk != 0.0f) ? 1.0f / pk : 0.0f;
#pragma unroll
        for (int lr = 0; lr < 4; ++lr) {
            const int i = 4 * lr + r;
            if (i > k) {
                const float l = e[lr][k] * rk;
#pragma unroll
                for (int j = 0; j < N; ++j)
                    if (j > k) e[lr][j] = fmaf(-l, prow[j], e[lr][j]);
            }
        }
    }
    logabs = near_identity ? log(fabs(prod)) : lsum;
    return ok;
}

__global__ void __launch_bounds__(THREADS, 2)
k16_chunk(KParams p, const float* __restrict__ x, float* __restrict__ S_out, float* __restrict__ totals,
          uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t chain0 = (int64_t)blockIdx.x * WARPS;

    // chain id -> (b, k, h), h fastest, so that a CTA's chains are the heads of
    // one token range: their slices are contiguous in memory.
    auto decode = [&](int64_t chain, int64_t& b, int64_t& k, int64_t& h) {
        h = chain % p.H;
        const int64_t bk = chain / p.H;
        k = bk % p.K;
        b = bk / p.K;
    };

    // ---- phase 1a: copy the CTA's slices into shared memory ----------------
    for (int g = tid; g < WARPS * CT * 64; g += THREADS) {
        const int w = g / (CT * 64), j = (g / 64) % CT, q16 = g % 64;
        const int64_t chain = chain0 + w;
        if (chain >= nchains) continue;
        int64_t b, k, h;
        decode(chain, b, k, h);
        const int64_t t = k * CT + j;
        if (t >= p.L) continue;
        const int row = q16 >> 2, col4 = q16 & 3;
        const float* src = x + (((b * p.L + t) * p.H + h) * NN) + row * N + col4 * 4;
        cp_async16(&sm.x[w][j][row * ROWW + col4 * 4], src);
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- phase 1b: per-token scalars (determinant scale) -------------------
    {
        const int grp = tid >> 2, r = tid & 3;       // 64 groups of 4 lanes
        const int w = grp / CT, j = grp % CT;
        const int64_t chain = chain0 + w;
        bool live = chain < nchains;
        int64_t b = 0, k = 0, h = 0;
        if (live) {
            decode(chain, b, k, h);
            live = k * CT + j < p.L;
        }
        float c = 1.0f, cm1 = 0.0f;
        if (p.mode == MRU_MODE_DETNORM) {
            float e[4][N];
            const float* xs = sm.x[w][j];
#pragma unroll
            for (int lr = 0; lr < 4; ++lr) {
                const int i = 4 * lr + r;
#pragma unroll
                for (int jj = 0; jj < N; ++jj) e[lr][jj] = live ? p.alpha * xs[i * ROWW + jj] : 0.0f;
            }
            double ld = 0.0;
            bool singular = false;
            bool ok = true;
            if (p.add_identity) ok = group_logabsdet(e, r, true, ld, singular);
            // every group of the warp must agree before the pivoted retry, as
            // the shuffles inside span the whole warp
            const bool retry = __any_sync(0xffffffffu, !p.add_identity || !ok);
            if (retry) {
                const bool need = !p.add_identity || !ok;
#pragma unroll
                for (int lr = 0; lr < 4; ++lr) {
                    const int i = 4 * lr + r;
#pragma unroll
                    for (int jj = 0; jj < N; ++jj)
                        e[lr][jj] = live ? p.alpha * xs[i * ROWW + jj] + ((p.add_identity && i == jj) ? 1.0f : 0.0f)
                                         : (i == jj ? 1.0f : 0.0f);
                }
                double ld2 = 0.0;
                bool sing2 = false;
                group_logabsdet(e, r, false, ld2, sing2);
                if (need) { ld = ld2; singular = sing2; }
            }
            const double cm1d = expm1(-ld / N);
            c = (float)(1.0 + cm1d);
            cm1 = (float)cm1d;
            if (live && (singular || !isfinite(ld) || !isfinite(c) || c == 0.0f)) {
                if (r == 0) atomicOr(status, STATUS_SINGULAR);
                c = 0.0f;
                cm1 = 0.0f;
            }
        }
        if (r == 0) {
            sm.c[w][j][0] = c;
            sm.c[w][j][1] = cm1;
        }
    }
    __syncthreads();

    // ---- phase 2: the chain of warp `warp` ---------------------------------
    const int64_t chain = chain0 + warp;
    if (chain >= nchains) return;
    int64_t b, k, h;
    decode(chain, b, k, h);
    const int g = lane >> 2, q = lane & 3;
    float Qd[2][4];                                  // accumulator layout, 2 column tiles
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) Qd[nt][i] = 0.0f;

    const float dconst = p.add_identity ? 0.0f : -1.0f;   // diagonal of F besides c-1
    for (int j = 0; j < CT; ++j) {
        const int64_t t = k * CT + j;
        if (t >= p.L) break;
        const float* xs = sm.x[warp][j];
        const float c = sm.c[warp][j][0];
        const float ca = c * p.alpha;
        const float dval = p.add_identity ? sm.c[warp][j][1] : dconst;
        auto F = [&](int rr, int cc) {
            const float v = ca * xs[rr * ROWW + cc];
            return (c == 0.0f) ? 0.0f : (rr == cc ? v + dval : v);
        };
        // B fragments of F with the permuted contraction index:
        // slot q <-> logical row 8kt + 2q, slot q + 4 <-> 8kt + 2q + 1.
        uint32_t bh[2][2][2], bl[2][2][2];
#pragma unroll
        for (int kt = 0; kt < 2; ++kt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                split_tf32(F(8 * kt + 2 * q, 8 * nt + g), bh[kt][nt][0], bl[kt][nt][0]);
                split_tf32(F(8 * kt + 2 * q + 1, 8 * nt + g), bh[kt][nt][1], bl[kt][nt][1]);
            }
        // A fragments straight from the state registers
        uint32_t ah[2][4], al[2][4];
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            split_tf32(Qd[kt][0], ah[kt][0], al[kt][0]);
            split_tf32(Qd[kt][2], ah[kt][1], al[kt][1]);
            split_tf32(Qd[kt][1], ah[kt][2], al[kt][2]);
            split_tf32(Qd[kt][3], ah[kt][3], al[kt][3]);
        }
        float acc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) mma_3xtf32(acc[nt], ah[kt], al[kt], bh[kt][nt], bl[kt][nt]);
        }
        float* out = S_out + (((b * p.L + t) * p.H + h) * NN);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int c0 = 8 * nt + 2 * q;
            Qd[nt][0] += F(g, c0) + acc[nt][0];
            Qd[nt][1] += F(g, c0 + 1) + acc[nt][1];
            Qd[nt][2] += F(g + 8, c0) + acc[nt][2];
            Qd[nt][3] += F(g + 8, c0 + 1) + acc[nt][3];
            *reinterpret_cast<float2*>(out + g * N + c0) = make_float2(Qd[nt][0], Qd[nt][1]);
            *reinterpret_cast<float2*>(out + (g + 8) * N + c0) = make_float2(Qd[nt][2], Qd[nt][3]);
        }
    }
    // chunk total, indexed (b*H + h)*K + k like the generic path
    float* tot = totals + ((b * p.H + h) * p.K + k) * NN;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int c0 = 8 * nt + 2 * q;
        *reinterpret_cast<float2*>(tot + g * N + c0) = make_float2(Qd[nt][0], Qd[nt][1]);
        *reinterpret_cast<float2*>(tot + (g + 8) * N + c0) = make_float2(Qd[nt][2], Qd[nt][3]);
    }
}

// S_t = C + C Q_t in place, one warp per chain.
__global__ void __launch_bounds__(THREADS)
k16_fixup(KParams p, const float* __restrict__ carry, float* __restrict__ S_out)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t chain = (int64_t)blockIdx.x * WARPS + warp;
    if (chain >= nchains) return;
    const int64_t h = chain % p.H, bk = chain / p.H, k = bk % p.K, b = bk / p.K;
    const int g = lane >> 2, q = lane & 3;
    const float* C = carry + ((b * p.H + h) * p.K + k) * NN;
    uint32_t ah[2][4], al[2][4];
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
        split_tf32(C[g * N + 8 * kt + q], ah[kt][0], al[kt][0]);
        split_tf32(C[(g + 8) * N + 8 * kt + q], ah[kt][1], al[kt][1]);
        split_tf32(C[g * N + 8 * kt + q + 4], ah[kt][2], al[kt][2]);
        split_tf32(C[(g + 8) * N + 8 * kt + q + 4], ah[kt][3], al[kt][3]);
    }
    float Cd[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int c0 = 8 * nt + 2 * q;
        Cd[nt][0] = C[g * N + c0];
        Cd[nt][1] = C[g * N + c0 + 1];
        Cd[nt][2] = C[(g + 8) * N + c0];
        Cd[nt][3] = C[(g + 8) * N + c0 + 1];
    }
    for (int j = 0; j < CT; ++j) {
        const int64_t t = k * CT + j;
        if (t >= p.L) break;
        float* Sq = S_out + (((b * p.L + t) * p.H + h) * NN);
        uint32_t bh[2][2][2], bl[2][2][2];
#pragma unroll
        for (int kt = 0; kt < 2; ++kt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                split_tf32(Sq[(8 * kt + q) * N + 8 * nt + g], bh[kt][nt][0], bl[kt][nt][0]);
                split_tf32(Sq[(8 * kt + q + 4) * N + 8 * nt + g], bh[kt][nt][1], bl[kt][nt][1]);
            }
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) mma_3xtf32(acc, ah[kt], al[kt], bh[kt][nt], bl[kt][nt]);
            const int c0 = 8 * nt + 2 * q;
            *reinterpret_cast<float2*>(Sq + g * N + c0) = make_float2(Cd[nt][0] + acc[0], Cd[nt][1] + acc[1]);
            *reinterpret_cast<float2*>(Sq + (g + 8) * N + c0) = make_float2(Cd[nt][2] + acc[2], Cd[nt][3] + acc[3]);
        }
    }
}

}  // namespace

int chunk_tokens() { return CT; }

bool supports(const KParams& p, bool readout)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_F32 && !readout &&
           (p.mode == MRU_MODE_RESHAPE || p.mode == MRU_MODE_DETNORM) && p.chunk == CT;
}

cudaError_t launch_chunk(const KParams& p, const float* x, float* S_out, float* totals, uint32_t* status,
                         cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    const unsigned grid = (unsigned)((nchains + WARPS - 1) / WARPS);
    const size_t sm = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(k16_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k16_chunk<<<grid, THREADS, sm, s>>>(p, x, S_out, totals, status);
    return cudaGetLastError();
}

cudaError_t launch_fixup(const KParams& p, const float* carry, float* S_out, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    const unsigned grid = (unsigned)((nchains + WARPS - 1) / WARPS);
    k16_fixup<<<grid, THREADS, 0, s>>>(p, carry, S_out);
    return cudaGetLastError();
}

}  // namespace n16
}  // namespace mru
