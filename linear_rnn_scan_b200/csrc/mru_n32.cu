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

#include <atomic>

#include "mru_internal.cuh"

namespace mru {
namespace n32 {
namespace {

constexpr int N = 32;
constexpr int NN = N * N;
constexpr int ROWB = 80;             // padded shared-memory row stride in bytes (32 bf16 + 16 B)
constexpr int SLICEB = N * ROWB;     // one token-head slice: 2,560 bytes
constexpr int SUB = n16::kSub;       // the chunk length is a multiple of it
constexpr int ST = 2;                // tokens per pipeline stage
constexpr int NS = 2;                // stages per warp: one in flight while one is consumed
constexpr int WARPS = 4;             // warps per CTA (4 CTAs per SM)
constexpr int THREADS = 32 * WARPS;

struct WarpSmem {
    unsigned char x[NS][ST][SLICEB]; // 10,240 bytes
    float dd[ST][2][N];              // D_i and D_i - 1 per token of the stage: 512 bytes
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int Pending>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(Pending));
}

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

// D = A B (+ 0).
__device__ __forceinline__ void mma_bf16_first(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
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
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            // the tile holds k in [16 kt, 16 kt + 15], n in [8 nt, 8 nt + 7]
            if (LOWER && 16 * kt + 15 <= 8 * nt) continue;      // no k > n
            if (!LOWER && 16 * kt >= 8 * nt + 7) continue;      // no k < n
            // the first tile a column tile meets starts its accumulator at zero
            const bool first = kt == 0 || (LOWER ? 15 <= 8 * nt : 0 >= 8 * nt + 7);   // tile (0, nt) skipped
            const uint32_t b0 = tri_mask(bm[kt][nt][0], 16 * kt - 8 * nt, d, LOWER);
            const uint32_t b1 = tri_mask(bm[kt][nt][1], 16 * kt + 8 - 8 * nt, d, LOWER);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                if (first) mma_bf16_first(acc[mt][nt], al[mt][kt], b0, b1);
                else mma_bf16(acc[mt][nt], al[mt][kt], b0, b1);
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

// D_i = exp(d tanh M_ii) and D_i - 1 (expm1) for the nt tokens of a stage
// (lane i: diagonal entry i).
__device__ __forceinline__ void stage_dd(const KParams& p, WarpSmem& ws, const unsigned char (*xs)[SLICEB], int nt,
                                         int lane)
{
    for (int j = 0; j < nt; ++j) {
        const uint16_t mb = *reinterpret_cast<const uint16_t*>(xs[j] + lane * ROWB + lane * 2);
        const float mii = __uint_as_float((uint32_t)mb << 16);
        const float dm1 = expm1f(p.ldu_d * tanhf(mii));
        ws.dd[j][0][lane] = 1.0f + dm1;
        ws.dd[j][1][lane] = dm1;
    }
    __syncwarp();
}

// chain id -> (b, k, h), h fastest (chain ids stay below 2^31).
struct Chain {
    int64_t b, h, k, tbeg, tend;
};
__device__ __forceinline__ Chain chain_at(const KParams& p, int64_t chain)
{
    Chain c;
    const uint32_t ci = (uint32_t)chain;
    const uint32_t bk = fastdiv(ci, p.h_mul, p.h_shr);
    const uint32_t b = fastdiv(bk, p.k_mul, p.k_shr);
    c.h = ci - bk * (uint32_t)p.H;
    c.k = bk - b * (uint32_t)p.K;
    c.b = b;
    c.tbeg = c.k * p.chunk;
    c.tend = (c.tbeg + p.chunk < p.L) ? c.tbeg + p.chunk : p.L;
    return c;
}

// The producer side of a warp's pipeline: the next stage of ST token slices
// (2 KB each, copied as 128 granules into rows padded to ROWB bytes) along
// the warp's chains w, w + W, ...
struct Feed {
    int64_t chain, stride, nchains, tok;
    int64_t t, tend;
    const uint16_t* xb;

    __device__ __forceinline__ void set(const KParams& p, const uint16_t* x)
    {
        if (chain >= nchains) return;
        const Chain c = chain_at(p, chain);
        xb = x + (c.b * p.L * p.H + c.h) * NN;
        t = c.tbeg;
        tend = c.tend;
    }
    // Copies the next stage into dst (nothing once the chains are done) and
    // commits a cp.async group either way.
    __device__ __forceinline__ void issue(unsigned char (*dst)[SLICEB], int lane, const KParams& p, const uint16_t* x)
    {
        if (chain < nchains) {
            const int nt = (tend - t < ST) ? (int)(tend - t) : ST;
#pragma unroll
            for (int i = 0; i < ST * 128 / 32; ++i) {
                const int gi = lane + 32 * i;
                const int j = gi >> 7, g16 = gi & 127, row = g16 >> 2, c4 = g16 & 3;
                if (j < nt) cp_async16(dst[j] + row * ROWB + c4 * 16, xb + (t + j) * tok + row * N + c4 * 8);
            }
            t += ST;
            if (t >= tend) {
                chain += stride;
                set(p, x);
            }
        }
        cp_async_commit();
    }
};

__global__ void __launch_bounds__(THREADS, 4)
k32_reduce(KParams p, const uint16_t* __restrict__ x, float* __restrict__ totals)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * WARPS + warp, stride = (int64_t)gridDim.x * WARPS;
    Feed feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = p.H * NN;
    feed.set(p, x);
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) feed.issue(ws.x[s], lane, p, x);
    int cs = 0, ps = NS - 1;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        State st;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) st[mt][nt][i] = 0.0f;
        for (int64_t t0 = c.tbeg; t0 < c.tend; t0 += ST) {
            feed.issue(ws.x[ps], lane, p, x);
            ps = (ps + 1 == NS) ? 0 : ps + 1;
            cp_async_wait<NS - 1>();
            __syncwarp();
            const int ntk = (c.tend - t0 < ST) ? (int)(c.tend - t0) : ST;
            stage_dd(p, ws, ws.x[cs], ntk, lane);
            for (int j = 0; j < ntk; ++j) apply_token<true>(st, ws.x[cs][j], ws.dd[j][0], ws.dd[j][1], p.ldu_a, lane);
            __syncwarp();
            cs = (cs + 1 == NS) ? 0 : cs + 1;
        }
        store_state(totals + ((c.b * p.H + c.h) * p.K + c.k) * NN, st, lane >> 2, lane & 3);
    }
}

// The chain's carry C = E1 (I + R0[k-1]) in fp64 (E1 alone for the first
// chunk of a group), computed straight into the accumulator layout from L2:
// lane (g, q) forms rows 16 mt + g + 8 h, columns 8 nt + 2 q (+ 1).
__device__ __forceinline__ void form_carry(const double* e1, const float* rp, int lane, State& st)
{
    const int g = lane >> 2, q = lane & 3;
    double acc[2][2][4][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const double2 v = *reinterpret_cast<const double2*>(e1 + (16 * mt + g + 8 * h) * N + 8 * nt + 2 * q);
                acc[mt][h][nt][0] = v.x;
                acc[mt][h][nt][1] = v.y;
            }
    if (rp) {
#pragma unroll 2
        for (int kk = 0; kk < N; ++kk) {
            double av[2][2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int h = 0; h < 2; ++h) av[mt][h] = e1[(16 * mt + g + 8 * h) * N + kk];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const float2 r = *reinterpret_cast<const float2*>(rp + kk * N + 8 * nt + 2 * q);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        acc[mt][h][nt][0] = fma(av[mt][h], (double)r.x, acc[mt][h][nt][0]);
                        acc[mt][h][nt][1] = fma(av[mt][h], (double)r.y, acc[mt][h][nt][1]);
                    }
            }
        }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                st[mt][nt][2 * h] = (float)acc[mt][h][nt][0];
                st[mt][nt][2 * h + 1] = (float)acc[mt][h][nt][1];
            }
}

// The carry of a single-chunk problem: S0 (fp32, from L2) or I.
__device__ __forceinline__ void direct_carry(const float* s0, int lane, State& st)
{
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = 16 * mt + g + 8 * h, col = 8 * nt + 2 * q;
                float2 v = make_float2(row == col ? 1.0f : 0.0f, row == col + 1 ? 1.0f : 0.0f);
                if (s0) v = *reinterpret_cast<const float2*>(s0 + row * N + col);
                st[mt][nt][2 * h] = v.x;
                st[mt][nt][2 * h + 1] = v.y;
            }
}

__global__ void __launch_bounds__(THREADS, 4)
k32_apply(KParams p, const uint16_t* __restrict__ x, const float* __restrict__ R0, const double* __restrict__ E1,
          int G, float* __restrict__ S_out, const float* __restrict__ S0, int direct)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * WARPS + warp, stride = (int64_t)gridDim.x * WARPS;
    const int g = lane >> 2, q = lane & 3;
    const int64_t tok = p.H * NN;
    const int64_t n1 = (p.K + G - 1) / G;
    Feed feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = tok;
    feed.set(p, x);
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) feed.issue(ws.x[s], lane, p, x);
    int cs = 0, ps = NS - 1;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        const int64_t seq = c.b * p.H + c.h;
        State st;
        if (direct)
            direct_carry(S0 ? S0 + seq * NN : nullptr, lane, st);
        else
            form_carry(E1 + (seq * n1 + c.k / G) * NN, (c.k % G) ? R0 + (seq * p.K + c.k - 1) * NN : nullptr, lane,
                       st);
        float* ob = S_out + (c.b * p.L * p.H + c.h) * NN;
        for (int64_t t0 = c.tbeg; t0 < c.tend; t0 += ST) {
            feed.issue(ws.x[ps], lane, p, x);
            ps = (ps + 1 == NS) ? 0 : ps + 1;
            cp_async_wait<NS - 1>();
            __syncwarp();
            const int ntk = (c.tend - t0 < ST) ? (int)(c.tend - t0) : ST;
            stage_dd(p, ws, ws.x[cs], ntk, lane);
            for (int j = 0; j < ntk; ++j) {
                apply_token<false>(st, ws.x[cs][j], ws.dd[j][0], ws.dd[j][1], p.ldu_a, lane);
                store_state(ob + (t0 + j) * tok, st, g, q);
            }
            __syncwarp();
            cs = (cs + 1 == NS) ? 0 : cs + 1;
        }
    }
}

// CTAs of a persistent launch: resident CTAs per SM times the SM count,
// cached per device and kernel slot; no more than the chains need.
std::atomic<int> g_resident[64][2];

cudaError_t persistent_grid(int slot, const void* kern, int64_t nchains, unsigned& grid)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int res = (dev >= 0 && dev < 64) ? g_resident[dev][slot].load(std::memory_order_relaxed) : 0;
    if (res <= 0) {
        int sms = 0, per_sm = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, sizeof(WarpSmem) * WARPS)) !=
            cudaSuccess)
            return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        res = sms * per_sm;
        if (dev >= 0 && dev < 64) g_resident[dev][slot].store(res, std::memory_order_relaxed);
    }
    const int64_t need = (nchains + WARPS - 1) / WARPS;
    grid = (unsigned)(need < res ? need : res);
    return cudaSuccess;
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
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(WarpSmem) * WARPS;
    cudaError_t e = cudaFuncSetAttribute(k32_reduce, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    if ((e = persistent_grid(0, (const void*)k32_reduce, nchains, grid)) != cudaSuccess) return e;
    k32_reduce<<<grid, THREADS, sm, s>>>(p, reinterpret_cast<const uint16_t*>(x), totals);
    return cudaGetLastError();
}

cudaError_t launch_apply(const KParams& p, const void* x, const carry::Plan& pl, const char* ws, float* S_out,
                         const float* S0, bool direct, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(WarpSmem) * WARPS;
    cudaError_t e = cudaFuncSetAttribute(k32_apply, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    if ((e = persistent_grid(1, (const void*)k32_apply, nchains, grid)) != cudaSuccess) return e;
    k32_apply<<<grid, THREADS, sm, s>>>(p, reinterpret_cast<const uint16_t*>(x),
                                        reinterpret_cast<const float*>(ws + pl.R[0]),
                                        reinterpret_cast<const double*>(ws + pl.E[1]), pl.G, S_out,
                                        direct ? S0 : nullptr, direct ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace n32
}  // namespace mru
