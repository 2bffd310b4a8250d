// mru_n32.cu -- n = 32 LDU-fill scan kernels on the tensor cores (bf16
// embeddings), two passes over the embeddings like the n = 16 path.
//
// The token matrix X = L D U (L = I + a strict_lower(M), U = I + a
// strict_upper(M), D = diag(exp(d tanh M_ii)); "Improving Matrix Recurrent
// Units as an Attention Alternative", LDU factor filling) is never formed:
// the chain applies the three factors one after the other, in identity-split
// form for the reduce pass (P = I + Q):
//     Q1 = Q + a (Ls + Q Ls)                 (P L,  Ls = strict_lower(M))
//     Q2 = Q1 D + (D - I)                    (P L D, a column scaling)
//     Q3 = Q2 + a (Us + Q2 Us)               (P L D U, Us = strict_upper(M))
// and on the full state for the apply pass (S L D U).  The two products per
// token run on mma.sync m16n8k16 with bf16 operands and fp32 accumulation:
// M's entries are bf16 already (exact operands, loaded with ldmatrix.trans);
// the state is split into bf16 hi + lo (two products).  Tiles of the
// triangular factors that are all zero are skipped.  D_i - 1 comes from
// expm1 so that the diagonal keeps its small deviation exactly.
#include <string.h>

#include "mru_internal.cuh"

namespace mru {
namespace n32 {
namespace {

constexpr int N = 32;
constexpr int NN = N * N;
constexpr int ROWB = 80;             // padded shared-memory row stride in bytes (32 bf16 + 16 B)
constexpr int SLICEB = N * ROWB;     // one token-head slice: 2,560 bytes
constexpr int SUB = n16::kSub;       // tokens per pass (the chunk length is a multiple)
constexpr int WARPS = 4;
constexpr int THREADS = 32 * WARPS;

struct WarpSmem {
    unsigned char x[SUB][SLICEB];    // 20,480 bytes
    float dd[SUB][2][N];             // D_i and D_i - 1 per token: 2,048 bytes
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::); }

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* smem_row)
{
    const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(smem_row));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

// D += A B, m16n8k16, bf16 operands, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 pair of (lo_elem, hi_elem), round to nearest.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Split a pair of fp32 values into bf16 hi and lo parts (x ~ hi + lo).
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo)
{
    hi = pack_bf16(x0, x1);
    lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

// The state: 32 x 32 fp32 in accumulator layout, st[mt][nt][i] holds
// element (16 mt + g + 8 (i >> 1), 8 nt + 2 q + (i & 1)).
using State = float[2][4][4];

// A fragments (hi, lo) of the state: the accumulator tile (mt, 2 kt) and
// (mt, 2 kt + 1) are exactly the A fragment (mt, kt) of m16n8k16.
__device__ __forceinline__ void state_frags(const State& st, uint32_t (&ah)[2][2][4], uint32_t (&al)[2][2][4])
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            split_pair(st[mt][2 * kt][0], st[mt][2 * kt][1], ah[mt][kt][0], al[mt][kt][0]);
            split_pair(st[mt][2 * kt][2], st[mt][2 * kt][3], ah[mt][kt][1], al[mt][kt][1]);
            split_pair(st[mt][2 * kt + 1][0], st[mt][2 * kt + 1][1], ah[mt][kt][2], al[mt][kt][2]);
            split_pair(st[mt][2 * kt + 1][2], st[mt][2 * kt + 1][3], ah[mt][kt][3], al[mt][kt][3]);
        }
}

// B fragments of M (K x N row-major bf16 in shared memory) for all (kt, nt):
// bm[kt][nt][h] holds rows k = 16 kt + 8 h + 2 q, + 1 of column n = 8 nt + g.
__device__ __forceinline__ void load_m_frags(const unsigned char* xs, int lane, uint32_t (&bm)[2][4][2])
{
    const int r = lane & 15, cg = lane >> 4;     // row within the 16-row k-tile, column-tile of the pair
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t v[4];
            ldsm_x4_trans(v, xs + (16 * kt + r) * ROWB + (8 * (2 * np + cg)) * 2);
            bm[kt][2 * np][0] = v[0];
            bm[kt][2 * np][1] = v[1];
            bm[kt][2 * np + 1][0] = v[2];
            bm[kt][2 * np + 1][1] = v[3];
        }
}

// Keep the bf16 halves of a B register whose (k, n) satisfy k > n (lower)
// or k < n (upper).  c = 16 kt + 8 h - 8 nt is the tile offset, d = 2 q - g.
__device__ __forceinline__ uint32_t tri_mask(uint32_t v, int c, int d, bool lower)
{
    const int lo_kn = c + d, hi_kn = c + d + 1;    // k - n of the two halves
    const bool keep_lo = lower ? lo_kn > 0 : lo_kn < 0;
    const bool keep_hi = lower ? hi_kn > 0 : hi_kn < 0;
    return v & ((keep_lo ? 0x0000ffffu : 0u) | (keep_hi ? 0xffff0000u : 0u));
}

// acc = state x T where T is the lower (Ls) or upper (Us) strict part of M;
// tiles of T that are all zero are skipped at compile time.
template <bool LOWER>
__device__ __forceinline__ void tri_product(const uint32_t (&ah)[2][2][4], const uint32_t (&al)[2][2][4],
                                            const uint32_t (&bm)[2][4][2], int d, State& acc)
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            // the tile holds k in [16 kt, 16 kt + 15], n in [8 nt, 8 nt + 7]
            if (LOWER && 16 * kt + 15 <= 8 * nt) continue;      // no k > n
            if (!LOWER && 16 * kt >= 8 * nt + 7) continue;      // no k < n
            const uint32_t b0 = tri_mask(bm[kt][nt][0], 16 * kt - 8 * nt, d, LOWER);
            const uint32_t b1 = tri_mask(bm[kt][nt][1], 16 * kt + 8 - 8 * nt, d, LOWER);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                mma_bf16(acc[mt][nt], al[mt][kt], b0, b1);
                mma_bf16(acc[mt][nt], ah[mt][kt], b0, b1);
            }
        }
}

// M at this lane's accumulator positions, as fp32 pairs (row 16 mt + g + 8 h,
// columns 8 nt + 2 q, + 1).
__device__ __forceinline__ void load_m_d(const unsigned char* xs, int g, int q, float (&md)[2][4][4])
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t v =
                    *reinterpret_cast<const uint32_t*>(xs + (16 * mt + g + 8 * h) * ROWB + (8 * nt + 2 * q) * 2);
                md[mt][nt][2 * h] = bf16_lo(v);
                md[mt][nt][2 * h + 1] = bf16_hi(v);
            }
}

// One token applied to the state.  split: state is Q = P - I (reduce pass)
// and the factors' identity parts enter as the extra terms; otherwise the
// state is the full product S (apply pass).
template <bool SPLIT>
__device__ __forceinline__ void apply_token(State& st, const unsigned char* xs, const float* Dv, const float* Dm1,
                                            float a, int lane)
{
    const int g = lane >> 2, q = lane & 3, d = 2 * q - g;
    uint32_t bm[2][4][2];
    load_m_frags(xs, lane, bm);
    float md[2][4][4];
    load_m_d(xs, g, q, md);
    uint32_t ah[2][2][4], al[2][2][4];
    State acc;
    // --- P L ---
    state_frags(st, ah, al);
    tri_product<true>(ah, al, bm, d, acc);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 16 * mt + g + 8 * (i >> 1), col = 8 * nt + 2 * q + (i & 1);
                const float ls = (row > col) ? md[mt][nt][i] : 0.0f;
                st[mt][nt][i] += a * ((SPLIT ? ls : 0.0f) + acc[mt][nt][i]);
            }
    // --- (P L) D ---
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const float2 dv = *reinterpret_cast<const float2*>(Dv + 8 * nt + 2 * q);
        const float2 dm = *reinterpret_cast<const float2*>(Dm1 + 8 * nt + 2 * q);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 16 * mt + g + 8 * (i >> 1), col = 8 * nt + 2 * q + (i & 1);
                float v = st[mt][nt][i] * ((i & 1) ? dv.y : dv.x);
                if (SPLIT && row == col) v += (i & 1) ? dm.y : dm.x;
                st[mt][nt][i] = v;
            }
    }
    // --- (P L D) U ---
    state_frags(st, ah, al);
    tri_product<false>(ah, al, bm, d, acc);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 16 * mt + g + 8 * (i >> 1), col = 8 * nt + 2 * q + (i & 1);
                const float us = (row < col) ? md[mt][nt][i] : 0.0f;
                st[mt][nt][i] += a * ((SPLIT ? us : 0.0f) + acc[mt][nt][i]);
            }
}

__device__ __forceinline__ void store_state(float* out, const State& st, int g, int q)
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<float2*>(out + (16 * mt + g + 8 * h) * N + 8 * nt + 2 * q) =
                    make_float2(st[mt][nt][2 * h], st[mt][nt][2 * h + 1]);
}

// Copy the pass's slices (2 KB each, 128 granules) and form D, D - 1.
__device__ __forceinline__ void load_pass(const KParams& p, WarpSmem& ws, const uint16_t* xb, int64_t tok, int64_t t0,
                                          int nt, int lane)
{
#pragma unroll
    for (int i = 0; i < SUB * 128 / 32; ++i) {
        const int gi = lane + 32 * i;
        const int j = gi >> 7, q16 = gi & 127, row = q16 >> 2, c4 = q16 & 3;
        if (j < nt) cp_async16(ws.x[j] + row * ROWB + c4 * 16, xb + (t0 + j) * tok + row * N + c4 * 8);
    }
    cp_async_wait_all();
    __syncwarp();
    for (int j = 0; j < nt; ++j) {
        const uint16_t mb = *reinterpret_cast<const uint16_t*>(ws.x[j] + lane * ROWB + lane * 2);
        const float mii = __uint_as_float((uint32_t)mb << 16);
        const float z = p.ldu_d * tanhf(mii);
        const float dm1 = expm1f(z);
        ws.dd[j][0][lane] = 1.0f + dm1;
        ws.dd[j][1][lane] = dm1;
    }
    __syncwarp();
}

struct ChainIx {
    int64_t b, h, k, tbeg, tend;
};
__device__ __forceinline__ ChainIx chain_ix(const KParams& p, int64_t chain)
{
    ChainIx c;
    c.h = chain % p.H;
    const int64_t bk = chain / p.H;
    c.k = bk % p.K;
    c.b = bk / p.K;
    c.tbeg = c.k * p.chunk;
    c.tend = (c.tbeg + p.chunk < p.L) ? c.tbeg + p.chunk : p.L;
    return c;
}

__global__ void __launch_bounds__(THREADS)
k32_reduce(KParams p, const uint16_t* __restrict__ x, float* __restrict__ totals)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem_raw)[warp];
    const int64_t chain = (int64_t)blockIdx.x * WARPS + warp;
    if (chain >= p.B * p.H * p.K) return;
    const ChainIx c = chain_ix(p, chain);
    const int64_t tok = p.H * NN;
    const uint16_t* xb = x + (c.b * p.L * p.H + c.h) * NN;
    State st;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) st[mt][nt][i] = 0.0f;
    for (int64_t t0 = c.tbeg; t0 < c.tend; t0 += SUB) {
        const int ntk = (c.tend - t0 < SUB) ? (int)(c.tend - t0) : SUB;
        load_pass(p, ws, xb, tok, t0, ntk, lane);
        for (int j = 0; j < ntk; ++j) apply_token<true>(st, ws.x[j], ws.dd[j][0], ws.dd[j][1], p.ldu_a, lane);
        __syncwarp();
    }
    store_state(totals + ((c.b * p.H + c.h) * p.K + c.k) * NN, st, lane >> 2, lane & 3);
}

__global__ void __launch_bounds__(THREADS)
k32_apply(KParams p, const uint16_t* __restrict__ x, const float* __restrict__ R0, const double* __restrict__ E1,
          int G, float* __restrict__ S_out)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem_raw)[warp];
    const int64_t chain = (int64_t)blockIdx.x * WARPS + warp;
    if (chain >= p.B * p.H * p.K) return;
    const ChainIx c = chain_ix(p, chain);
    const int64_t seq = c.b * p.H + c.h;
    const int g = lane >> 2, q = lane & 3;
    State st;
    // carry C = E1 (I + R0[k-1]) in fp64, each lane a 4 x 8 block, staged in
    // the x buffer (8 KB of E1, 4 KB of C)
    {
        double* sE = reinterpret_cast<double*>(ws.x[0]);
        float* sC = reinterpret_cast<float*>(ws.x[4]);
        const int64_t n1 = (p.K + G - 1) / G;
        const double* e1 = E1 + (seq * n1 + c.k / G) * NN;
        for (int e = lane; e < NN; e += 32) sE[e] = e1[e];
        __syncwarp();
        const int r0 = (lane >> 2) * 4, c0 = (lane & 3) * 8;
        double acc[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) acc[i][cc] = sE[(r0 + i) * N + c0 + cc];
        if (c.k % G != 0) {
            const float* rp = R0 + (seq * p.K + c.k - 1) * NN;
#pragma unroll 2
            for (int kk = 0; kk < N; ++kk) {
                const float4 r1 = *reinterpret_cast<const float4*>(rp + kk * N + c0);
                const float4 r2 = *reinterpret_cast<const float4*>(rp + kk * N + c0 + 4);
                const double bv[8] = {r1.x, r1.y, r1.z, r1.w, r2.x, r2.y, r2.z, r2.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double av = sE[(r0 + i) * N + kk];
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) acc[i][cc] = fma(av, bv[cc], acc[i][cc]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) sC[(r0 + i) * N + c0 + cc] = (float)acc[i][cc];
        __syncwarp();
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float2 v = *reinterpret_cast<const float2*>(sC + (16 * mt + g + 8 * h) * N + 8 * nt + 2 * q);
                    st[mt][nt][2 * h] = v.x;
                    st[mt][nt][2 * h + 1] = v.y;
                }
        __syncwarp();
    }
    const int64_t tok = p.H * NN;
    const uint16_t* xb = x + (c.b * p.L * p.H + c.h) * NN;
    float* ob = S_out + (c.b * p.L * p.H + c.h) * NN;
    for (int64_t t0 = c.tbeg; t0 < c.tend; t0 += SUB) {
        const int ntk = (c.tend - t0 < SUB) ? (int)(c.tend - t0) : SUB;
        load_pass(p, ws, xb, tok, t0, ntk, lane);
        for (int j = 0; j < ntk; ++j) {
            apply_token<false>(st, ws.x[j], ws.dd[j][0], ws.dd[j][1], p.ldu_a, lane);
            store_state(ob + (t0 + j) * tok, st, g, q);
        }
        __syncwarp();
    }
}

}  // namespace

bool supports(const KParams& p, bool readout)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_BF16 && !readout && p.mode == MRU_MODE_LDU &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_BF16X3) && p.chunk > 0 && p.chunk % SUB == 0;
}

int32_t preferred_chunk(int64_t token_heads)
{
    int32_t m = 1;
    while (m < 16 && token_heads / ((int64_t)SUB * 2 * m) >= 8192) m *= 2;
    return SUB * m;
}

cudaError_t launch_reduce(const KParams& p, const void* x, float* totals, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    const unsigned grid = (unsigned)((nchains + WARPS - 1) / WARPS);
    const size_t sm = sizeof(WarpSmem) * WARPS;
    cudaError_t e = cudaFuncSetAttribute(k32_reduce, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k32_reduce<<<grid, THREADS, sm, s>>>(p, reinterpret_cast<const uint16_t*>(x), totals);
    return cudaGetLastError();
}

cudaError_t launch_apply(const KParams& p, const void* x, const carry::Plan& pl, const char* ws, float* S_out,
                         cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    const unsigned grid = (unsigned)((nchains + WARPS - 1) / WARPS);
    const size_t sm = sizeof(WarpSmem) * WARPS;
    cudaError_t e = cudaFuncSetAttribute(k32_apply, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k32_apply<<<grid, THREADS, sm, s>>>(p, reinterpret_cast<const uint16_t*>(x),
                                        reinterpret_cast<const float*>(ws + pl.R[0]),
                                        reinterpret_cast<const double*>(ws + pl.E[1]), pl.G, S_out);
    return cudaGetLastError();
}

}  // namespace n32
}  // namespace mru
