// mru_n64_bwd.cu -- backward (vector-Jacobian product) of the n = 64 scan on
// the tensor cores, for tf32 arithmetic (mru_problem.math = MRU_MATH_TF32),
// fp32 embeddings, reshape or determinant-corrected construction.
//
// The chain rule of S_t = S_{t-1} X_t, as in the generic backward: with
// G_t = dL/dS_t (every later state included), G_{t-1} = dS_{t-1} + G_t X_t^T,
// dL/dX_t = S_{t-1}^T G_t and dL/dS0 = G_1 X_1^T.  Chunked the same way; one
// CTA of 4 warps per chunk, warp w owning rows 16 w .. 16 w + 15 of every
// 64 x 64 matrix; every product on mma.sync m16n8k8 tf32 with fp32
// accumulation, the forward's arithmetic:
//   k64b_local   right to left through the chunk with a zero gradient
//                entering: the chunk's local gradient G and T = W^T - I with
//                W = X_{t0+1} ... X_{t1}, both in registers.  G <- dS + G + G F^T
//                and T <- T + F^T + T F^T take the same B operand, F^T =
//                c alpha M^T + (c - 1) I (F = X - I, M the raw slice).
//   (the chunk-gradient scan between the passes is the generic one)
//   k64b_apply   right to left from the gradient entering the chunk: G in
//                shared memory (dX = S_{t-1}^T G needs all of its rows in
//                every warp), dX in registers, then the construction's chain
//                rule to the embedding gradient: reshape alpha dX;
//                determinant-corrected alpha c (dX - <dX, Xr> Xr^-T / 64).
// The determinant scale c = |det Xr|^(-1/64), Xr = I + E, E = alpha M, comes
// from the trace series of log det (I + E) as in the forward kernel, here from
// the products P2 = (M^T)^2 and P3 = (M^T)^3 (traces and Frobenius norms do not
// change under transposition), and the same products give the inverse:
// Xr^-T = I - E^T + (E^T)^2 - (E^T)^3 + R with |R|_F <= |E^3|_F |E|_F / (1 - |E|_F).
// Where the series' certificate or that bound fails (far from the identity,
// or no identity in the construction), a pivoted Gauss-Jordan elimination in
// shared memory gives log|det| (fp64 sum) and the inverse.
#include "mru_internal.cuh"

namespace mru {
namespace n64 {
namespace {

constexpr int N = 64;
constexpr int NN = N * N;
constexpr int ROWW = 68;             // padded shared-memory row stride in words
constexpr int THREADS = 128;
constexpr int BUF = N * ROWW;        // floats in one padded 64 x 64 buffer

// Scratch of the reductions and of the pivoted elimination.
struct Common {
    float prow[2][N];                // pivot row (of W and of its inverse)
    float pcol[N];                   // multipliers of the pivot column
    float red[4][8];                 // per-warp partial traces and norms
    float red2[4];                   // per-warp partial <dX, Xr>
    double dsum;                     // log|det| of the pivoted elimination
    int flag;
    int piv;
};

struct LocalSmem {
    Common c;
    float x[2][BUF];                 // slices: this token's and the next one's
    float ds[2][BUF];                // dS_{t-1}, each warp its own 16 rows, double-buffered by token parity
};

struct ApplySmem {
    Common c;
    float x[2][BUF];                 // slices
    float s[BUF];                    // S_{t-1}; the pivoted inverse after dX has been formed
    float g[BUF];                    // G_t
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;\n" ::); }

// v rounded to the nearest tf32, ties away from zero (as cvt.rna.tf32.f32
// gives for finite v).
__device__ __forceinline__ uint32_t to_tf32(float v) { return (__float_as_uint(v) + 0x1000u) & 0xffffe000u; }

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 pair, `lo` in the low half, round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void zero(float (&a)[8][4])
{
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) a[nt][i] = 0.0f;
}

// Copies a 64 x 64 matrix (rows 64 floats apart in global memory) into a
// padded buffer, rows r_lo .. r_lo + nrows - 1, by the threads t_lo ..
// t_lo + nthr - 1 (cp.async; the caller commits).
__device__ __forceinline__ void issue_rows(float* dst, const float* src, int r_lo, int nrows, int t, int nthr)
{
    for (int gi = t; gi < nrows * 16; gi += nthr) {
        const int row = r_lo + (gi >> 4), c4 = gi & 15;
        cp_async16(dst + row * ROWW + 4 * c4, src + row * N + 4 * c4);
    }
}

// bf16 B fragment of M^T for k-tile kt (16 contraction rows) and column tile
// nt: B[k][n] = M[n][k], so both halves are adjacent in row 8 nt + g of M.
__device__ __forceinline__ void frag_mt16(const float* xs, int kt, int nt, int g, int q, uint32_t& b0, uint32_t& b1)
{
    const float2 u0 = *reinterpret_cast<const float2*>(xs + (8 * nt + g) * ROWW + 16 * kt + 2 * q);
    const float2 u1 = *reinterpret_cast<const float2*>(xs + (8 * nt + g) * ROWW + 16 * kt + 8 + 2 * q);
    b0 = pack_bf16(u0.x, u0.y);
    b1 = pack_bf16(u1.x, u1.y);
}

// tf32 B fragment of M^T for k-tile kt and column tile nt with the contraction
// index permuted as for accumulator-resident A operands (slot q <-> k =
// 8 kt + 2 q, slot q + 4 <-> k = 8 kt + 2 q + 1): b0 = M[8 nt + g][8 kt + 2 q], b1
// the next column.
__device__ __forceinline__ void frag_mt(const float* xs, int kt, int nt, int g, int q, uint32_t& b0, uint32_t& b1)
{
    const float2 m = *reinterpret_cast<const float2*>(xs + (8 * nt + g) * ROWW + 8 * kt + 2 * q);
    b0 = to_tf32(m.x);
    b1 = to_tf32(m.y);
}

// A fragment of k-tile kt from accumulator tiles (the permuted contraction).
__device__ __forceinline__ void frag_acc(const float (&A)[8][4], int kt, uint32_t (&a)[4])
{
    a[0] = to_tf32(A[kt][0]);
    a[1] = to_tf32(A[kt][2]);
    a[2] = to_tf32(A[kt][1]);
    a[3] = to_tf32(A[kt][3]);
}

struct Series {
    float cm1;                       // c - 1 (valid when ok)
    bool ok;                         // the series' certificate holds
    bool inv_ok;                     // ... and the inverse's three-term bound too
};

// The determinant scale from the trace series of log det(I + E), E = alpha M,
// by this CTA (all threads call; one barrier):
//   log det = tr E - tr E^2 / 2 + tr E^3 / 3 - tr E^4 / 4 + R,
//   |R| <= |E^3|_F |E^2|_F / (5 (1 - |E|_F)),
// taken when that bound is at most 1e-6, like the forward kernel.  The
// products are P2 = (M^T)^2 and P3 = P2 M^T (bf16 operands, fp32 accumulate):
// tr M^3 = <P2, M> and tr M^4 = <P3, M>.  With WantY, Y = (E^T)^2 - (E^T)^3 =
// alpha^2 P2 - alpha^3 P3 at this thread's accumulator positions when
// inv_ok: the inverse's terms beyond I - E^T, the dropped tail bounded by
// |E^3|_F |E|_F / (1 - |E|_F) <= 1e-3.
template <bool WantY>
__device__ __forceinline__ Series det_series(Common& cm, const float* xs, float alpha, int warp, int lane,
                                             float (&Y)[8][4])
{
    const int g = lane >> 2, q = lane & 3, r0 = 16 * warp;
    float (&P2)[8][4] = Y;
    zero(P2);
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
        // A[i][k] = M[k][i]: a column of M a register pair
        uint32_t a[4];
        const float* c0 = xs + (16 * kt + 2 * q) * ROWW + r0 + g;
        a[0] = pack_bf16(c0[0], c0[ROWW]);
        a[1] = pack_bf16(c0[8], c0[ROWW + 8]);
        a[2] = pack_bf16(c0[8 * ROWW], c0[9 * ROWW]);
        a[3] = pack_bf16(c0[8 * ROWW + 8], c0[9 * ROWW + 8]);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            uint32_t b0, b1;
            frag_mt16(xs, kt, nt, g, q, b0, b1);
            mma_bf16(P2[nt], a, b0, b1);
        }
    }
    float tr1 = 0.0f, tr2 = 0.0f, tr3 = 0.0f, tr4 = 0.0f, n1 = 0.0f, n2 = 0.0f, n3 = 0.0f;
    if (lane < 16) tr1 = xs[(r0 + lane) * ROWW + r0 + lane];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
            const float2 mv = *reinterpret_cast<const float2*>(xs + row * ROWW + col);
            const float mt0 = xs[col * ROWW + row], mt1 = xs[(col + 1) * ROWW + row];
            tr2 = fmaf(mv.x, mt0, fmaf(mv.y, mt1, tr2));
            tr3 = fmaf(P2[nt][2 * h8], mv.x, fmaf(P2[nt][2 * h8 + 1], mv.y, tr3));
            n1 = fmaf(mv.x, mv.x, fmaf(mv.y, mv.y, n1));
            n2 = fmaf(P2[nt][2 * h8], P2[nt][2 * h8], fmaf(P2[nt][2 * h8 + 1], P2[nt][2 * h8 + 1], n2));
        }
    // P3 = P2 M^T: all of it when the inverse wants it, else four column tiles at a time
    constexpr int HALVES = WantY ? 1 : 2;
    constexpr int TILES = 8 / HALVES;
    float P3[WantY ? 8 : 4][4];
#pragma unroll
    for (int hh = 0; hh < HALVES; ++hh) {
#pragma unroll
        for (int j = 0; j < TILES; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) P3[j][i] = 0.0f;
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            // accumulator tiles 2 kt, 2 kt + 1 are the bf16 A fragment of k-tile kt
            uint32_t a[4];
            a[0] = pack_bf16(P2[2 * kt][0], P2[2 * kt][1]);
            a[1] = pack_bf16(P2[2 * kt][2], P2[2 * kt][3]);
            a[2] = pack_bf16(P2[2 * kt + 1][0], P2[2 * kt + 1][1]);
            a[3] = pack_bf16(P2[2 * kt + 1][2], P2[2 * kt + 1][3]);
#pragma unroll
            for (int j = 0; j < TILES; ++j) {
                uint32_t b0, b1;
                frag_mt16(xs, kt, TILES * hh + j, g, q, b0, b1);
                mma_bf16(P3[j], a, b0, b1);
            }
        }
#pragma unroll
        for (int j = 0; j < TILES; ++j)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const int row = r0 + g + 8 * h8, col = 8 * (TILES * hh + j) + 2 * q;
                const float2 mv = *reinterpret_cast<const float2*>(xs + row * ROWW + col);
                tr4 = fmaf(P3[j][2 * h8], mv.x, fmaf(P3[j][2 * h8 + 1], mv.y, tr4));
                n3 = fmaf(P3[j][2 * h8], P3[j][2 * h8], fmaf(P3[j][2 * h8 + 1], P3[j][2 * h8 + 1], n3));
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
        float* rd = cm.red[warp];
        rd[0] = tr1; rd[1] = tr2; rd[2] = tr3; rd[3] = tr4; rd[4] = n1; rd[5] = n2; rd[6] = n3;
    }
    __syncthreads();
    float v[7];
#pragma unroll
    for (int i = 0; i < 7; ++i) v[i] = (cm.red[0][i] + cm.red[1][i]) + (cm.red[2][i] + cm.red[3][i]);
    const float a = alpha, a2 = a * a, a3 = a2 * a;
    const float ld = a * v[0] - a2 * (0.5f * v[1]) + a3 * (v[2] * (1.0f / 3.0f)) - a2 * a2 * (0.25f * v[3]);
    const float fe = a * sqrtf(v[4]), fe2 = a2 * sqrtf(v[5]), fe3 = a3 * sqrtf(v[6]);
    Series r;
    r.ok = fe < 1.0f && fe3 * fe2 / (5.0f * (1.0f - fe)) <= 1e-6f;    // false for non-finite inputs too
    r.inv_ok = r.ok && fe3 * fe / (1.0f - fe) <= 1e-3f;
    r.cm1 = r.ok ? expm1f(-ld * (1.0f / N)) : 0.0f;
    if constexpr (WantY) {
        if (r.inv_ok) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) Y[nt][i] = a2 * P2[nt][i] - a3 * P3[nt][i];
        }
    }
    return r;
}

// log|det W| of W = add_identity I + alpha M by elimination with partial
// pivoting, formed over the slice buffer W (destroyed: the caller reloads
// it).  With Winv, Gauss-Jordan: Winv ends as W^-1; without, only the rows
// below each pivot are eliminated.  NaN when a pivot column is zero.  All
// threads call.
__device__ double pivoted_logdet(Common& cm, float* W, float* Winv, float alpha, int add_identity)
{
    const int t = threadIdx.x;
    for (int e = t; e < NN; e += THREADS) {
        const int i = e >> 6, j = e & 63;
        float v = alpha * W[i * ROWW + j];
        if (add_identity && i == j) v += 1.0f;
        W[i * ROWW + j] = v;
        if (Winv) Winv[i * ROWW + j] = (i == j) ? 1.0f : 0.0f;
    }
    if (t == 0) { cm.dsum = 0.0; cm.flag = 0; }
    __syncthreads();
    for (int k = 0; k < N; ++k) {
        if (t < 32) {
            float best = -1.0f;
            int bi = k;
            for (int i = k + t; i < N; i += 32) {
                const float v = fabsf(W[i * ROWW + k]);
                if (v > best) { best = v; bi = i; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_down_sync(0xffffffffu, best, o);
                const int oi = __shfl_down_sync(0xffffffffu, bi, o);
                if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            if (t == 0) {
                cm.piv = bi;
                if (!(best > 0.0f)) cm.flag = 1;
            }
        }
        __syncthreads();
        const int piv = cm.piv;
        // the pivot row (after the swap) and the multipliers of column k
        for (int j = t; j < N; j += THREADS) {
            cm.prow[0][j] = W[piv * ROWW + j];
            if (Winv) cm.prow[1][j] = Winv[piv * ROWW + j];
        }
        const float pk = W[piv * ROWW + k];
        const float r = (pk != 0.0f) ? 1.0f / pk : 0.0f;
        if (t < N) {
            const int i = t == k ? piv : (t == piv ? k : t);     // row t after the swap
            cm.pcol[t] = W[i * ROWW + k] * r;
        }
        if (t == 0) cm.dsum += log(fabs((double)pk));
        __syncthreads();
        if (piv != k)                                             // old row k moves to row piv
            for (int j = t; j < N; j += THREADS) {
                W[piv * ROWW + j] = W[k * ROWW + j];
                if (Winv) Winv[piv * ROWW + j] = Winv[k * ROWW + j];
            }
        __syncthreads();
        for (int e = t; e < NN; e += THREADS) {
            const int i = e >> 6, j = e & 63;
            if (i == k) {
                W[i * ROWW + j] = cm.prow[0][j] * r;
                if (Winv) Winv[i * ROWW + j] = cm.prow[1][j] * r;
            } else if (Winv || i > k) {
                const float l = cm.pcol[i];
                W[i * ROWW + j] = fmaf(-l, cm.prow[0][j], W[i * ROWW + j]);
                if (Winv) Winv[i * ROWW + j] = fmaf(-l, cm.prow[1][j], Winv[i * ROWW + j]);
            }
        }
        __syncthreads();
    }
    const double ld = cm.dsum;
    const bool bad = cm.flag != 0;
    __syncthreads();
    return bad ? __longlong_as_double(0x7ff8000000000000ll) : ld;
}

// Plain reload of a slice after the elimination has overwritten it.
__device__ __forceinline__ void reload_slice(float* xs, const float* src)
{
    for (int gi = threadIdx.x; gi < NN / 4; gi += THREADS) {
        const int row = gi >> 4, c4 = gi & 15;
        *reinterpret_cast<float4*>(xs + row * ROWW + 4 * c4) = *reinterpret_cast<const float4*>(src + row * N + 4 * c4);
    }
    __syncthreads();
}

// A token's F = ca M + dv I and the determinant scale c.
struct Scale {
    float ca, dv;                    // F = ca M + dv I
    float c;                         // determinant scale (1 for reshape, 0 when singular)
};

// The scale from c - 1 (cm1, from the series or the pivoted elimination;
// good: the elimination found no zero pivot); SINGULAR is recorded, and F = 0,
// where c does not exist.
__device__ __forceinline__ Scale finish_scale(const KParams& p, bool detnorm, float cm1, bool good, uint32_t* status)
{
    Scale s;
    if (!detnorm) {
        s.ca = p.alpha;
        s.dv = p.add_identity ? 0.0f : -1.0f;
        s.c = 1.0f;
        return s;
    }
    const float c = 1.0f + cm1;
    if (!good || !isfinite(cm1) || !(c > 0.0f)) {
        if (threadIdx.x == 0) atomicOr(status, STATUS_SINGULAR);
        s.ca = 0.0f;
        s.dv = 0.0f;
        s.c = 0.0f;
    } else {
        s.ca = c * p.alpha;
        s.dv = p.add_identity ? cm1 : -1.0f;
        s.c = c;
    }
    return s;
}

// ---- local pass ---------------------------------------------------------------

__global__ void __launch_bounds__(THREADS, 2)
k64b_local(KParams p, const float* __restrict__ x, const float* __restrict__ dS, float* __restrict__ gloc,
           float* __restrict__ Wq, uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    LocalSmem& sm = *reinterpret_cast<LocalSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int r0 = 16 * warp;
    const int64_t chain = blockIdx.x;                // (b*H + h)*K + k, like the generic kernels
    const int64_t k = chain % p.K, bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    const bool more = t1 < p.L;                      // a chunk follows: W is needed
    const int64_t tok = p.H * NN;
    const int64_t base = (b * p.L * p.H + h) * NN;   // token 0 of this (b, h)
    const bool detnorm = p.mode == MRU_MODE_DETNORM;
    const bool series = detnorm && p.add_identity != 0;
    const int64_t tf = more ? t1 : t1 - 1;           // first token walked; down to t0 + 1

    float G[8][4], T[8][4];
    {
        const float* d0 = dS + base + (t1 - 1) * tok;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const float2 v = *reinterpret_cast<const float2*>(d0 + (r0 + g + 8 * h8) * N + 8 * nt + 2 * q);
                G[nt][2 * h8] = v.x;
                G[nt][2 * h8 + 1] = v.y;
            }
    }
    zero(T);
    if (tf > t0) {
        issue_rows(sm.x[0], x + base + tf * tok, 0, N, tid, THREADS);
        cp_commit();
        if (!more) {                                 // dS_{t1-2} for token t1 - 1, this warp's rows
            issue_rows(sm.ds[(t1 - 1) & 1], dS + base + (t1 - 2) * tok, r0, 16, lane, 32);
            cp_commit();
        }
    }
    int cur = 0;
    for (int64_t tau = tf; tau > t0; --tau, cur ^= 1) {
        float* xs = sm.x[cur];
        cp_wait_all();
        __syncthreads();
        if (tau - 1 > t0) {
            issue_rows(sm.x[cur ^ 1], x + base + (tau - 1) * tok, 0, N, tid, THREADS);
            cp_commit();
            if (tau - 1 < t1) {                      // dS_{tau-2} for token tau - 1
                issue_rows(sm.ds[(tau - 1) & 1], dS + base + (tau - 2) * tok, r0, 16, lane, 32);
                cp_commit();
            }
        }
        // ---- F = ca M + dv I ----
        float cm1 = 0.0f;
        bool good = true;
        if (detnorm) {
            float Yd[8][4];
            Series sr;
            sr.ok = false;
            sr.inv_ok = false;
            sr.cm1 = 0.0f;
            if (series) sr = det_series<false>(sm.c, xs, p.alpha, warp, lane, Yd);
            cm1 = sr.cm1;
            if (!sr.ok) {
                const double ld = pivoted_logdet(sm.c, xs, nullptr, p.alpha, p.add_identity);
                reload_slice(xs, x + base + tau * tok);
                good = isfinite(ld);
                cm1 = (float)expm1(-ld / N);
            }
        }
        const Scale sc = finish_scale(p, detnorm, cm1, good, status);
        if (tau == t1) {
            // T = F_{t1}^T
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q + e;
                        T[nt][2 * h8 + e] = fmaf(sc.ca, xs[col * ROWW + row], row == col ? sc.dv : 0.0f);
                    }
            continue;
        }
        // ---- G <- dS + G + G F^T, then T <- T + F^T + T F^T, F^T = ca M^T + dv I
        // (one product at a time: the B fragments are loaded twice, the
        // registers hold G, T and one accumulator) ----
        const float* dsb = sm.ds[tau & 1];
        {
            float aG[8][4];
            zero(aG);
#pragma unroll
            for (int kt = 0; kt < 8; ++kt) {
                uint32_t a[4];
                frag_acc(G, kt, a);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    uint32_t b0, b1;
                    frag_mt(xs, kt, nt, g, q, b0, b1);
                    mma_tf32(aG[nt], a, b0, b1);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                    const float2 dv2 = *reinterpret_cast<const float2*>(dsb + row * ROWW + col);
                    // G_{tau-1} = dS_{tau-1} + G X_tau^T
                    G[nt][2 * h8] = dv2.x + (G[nt][2 * h8] + fmaf(sc.ca, aG[nt][2 * h8], sc.dv * G[nt][2 * h8]));
                    G[nt][2 * h8 + 1] =
                        dv2.y + (G[nt][2 * h8 + 1] + fmaf(sc.ca, aG[nt][2 * h8 + 1], sc.dv * G[nt][2 * h8 + 1]));
                }
        }
        if (more) {
            float aT[8][4];
            zero(aT);
#pragma unroll
            for (int kt = 0; kt < 8; ++kt) {
                uint32_t a[4];
                frag_acc(T, kt, a);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    uint32_t b0, b1;
                    frag_mt(xs, kt, nt, g, q, b0, b1);
                    mma_tf32(aT[nt], a, b0, b1);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q + e, i = 2 * h8 + e;
                        // T <- T + F^T + T F^T (W <- X_tau W)
                        const float ft = fmaf(sc.ca, xs[col * ROWW + row], row == col ? sc.dv : 0.0f);
                        T[nt][i] = T[nt][i] + (ft + fmaf(sc.ca, aT[nt][i], sc.dv * T[nt][i]));
                    }
        }
    }
    cp_wait_all();
    float* go = gloc + chain * NN;
    float* wo = Wq + chain * NN;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
            *reinterpret_cast<float2*>(go + row * N + col) = make_float2(G[nt][2 * h8], G[nt][2 * h8 + 1]);
            // W - I = T^T
            wo[col * N + row] = more ? T[nt][2 * h8] : 0.0f;
            wo[(col + 1) * N + row] = more ? T[nt][2 * h8 + 1] : 0.0f;
        }
}

// ---- apply pass -----------------------------------------------------------------

// The state before token t into the S buffer: S_fwd at t - 1, S0 or I at t = 0.
__device__ __forceinline__ void issue_state(float* dst, const KParams& p, const float* S_fwd, const float* S0,
                                            int64_t base, int64_t tok, int64_t bh, int64_t t)
{
    if (t > 0) {
        issue_rows(dst, S_fwd + base + (t - 1) * tok, 0, N, threadIdx.x, THREADS);
    } else if (S0) {
        issue_rows(dst, S0 + bh * NN, 0, N, threadIdx.x, THREADS);
    } else {
        for (int e = threadIdx.x; e < NN; e += THREADS) dst[(e >> 6) * ROWW + (e & 63)] = (e >> 6) == (e & 63) ? 1.0f : 0.0f;
    }
    cp_commit();
}

__global__ void __launch_bounds__(THREADS, 2)
k64b_apply(KParams p, const float* __restrict__ x, const float* __restrict__ S0, const float* __restrict__ S_fwd,
           const float* __restrict__ dS, const float* __restrict__ Gin, float* __restrict__ dx,
           float* __restrict__ dS0, uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ApplySmem& sm = *reinterpret_cast<ApplySmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int r0 = 16 * warp;
    const int64_t chain = blockIdx.x;
    const int64_t k = chain % p.K, bh = chain / p.K;
    const int64_t h = bh % p.H, b = bh / p.H;
    const int64_t t0 = k * p.chunk;
    const int64_t t1 = (t0 + p.chunk < p.L) ? t0 + p.chunk : p.L;
    const bool has_in = t1 < p.L;                    // a gradient enters from the next chunk
    const int64_t tok = p.H * NN;
    const int64_t base = (b * p.L * p.H + h) * NN;
    const bool detnorm = p.mode == MRU_MODE_DETNORM;
    const bool series = detnorm && p.add_identity != 0;
    const int64_t tf = has_in ? t1 : t1 - 1;         // first token walked; down to t0

    issue_rows(sm.x[0], x + base + tf * tok, 0, N, tid, THREADS);
    issue_rows(sm.g, has_in ? Gin + chain * NN : dS + base + (t1 - 1) * tok, 0, N, tid, THREADS);
    cp_commit();
    issue_state(sm.s, p, S_fwd, S0, base, tok, bh, t1 - 1);    // for the first output token
    int cur = 0;
    for (int64_t tau = tf; tau >= t0; --tau, cur ^= 1) {
        float* xs = sm.x[cur];
        cp_wait_all();
        __syncthreads();
        if (tau > t0) {
            issue_rows(sm.x[cur ^ 1], x + base + (tau - 1) * tok, 0, N, tid, THREADS);
            cp_commit();
        }
        const bool out_tok = tau < t1;
        // dS_{tau-1} at this thread's accumulator positions (used last)
        float2 dsr[8][2];
        {
            const float* d0 = dS + base + (tau - 1) * tok;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8)
                    dsr[nt][h8] = tau > t0 ? *reinterpret_cast<const float2*>(d0 + (r0 + g + 8 * h8) * N + 8 * nt + 2 * q)
                                           : make_float2(0.0f, 0.0f);
        }
        // ---- dX = S_{tau-1}^T G, and this warp's part of <dX, Xr> ----
        float D[8][4];
        if (out_tok) {
            zero(D);
#pragma unroll
            for (int kt = 0; kt < 8; ++kt) {
                // A[i][k] = S[k][i], permuted contraction: slot q <-> k = 8 kt + 2 q
                uint32_t a[4];
                const float* sc0 = sm.s + (8 * kt + 2 * q) * ROWW + r0 + g;
                a[0] = to_tf32(sc0[0]);
                a[1] = to_tf32(sc0[8]);
                a[2] = to_tf32(sc0[ROWW]);
                a[3] = to_tf32(sc0[ROWW + 8]);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const float* gc = sm.g + (8 * kt + 2 * q) * ROWW + 8 * nt + g;
                    mma_tf32(D[nt], a, to_tf32(gc[0]), to_tf32(gc[ROWW]));
                }
            }
            if (detnorm) {
                // <dX, Xr> over this warp's rows, Xr = add_identity I + alpha M
                float part = 0.0f;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                        const float2 mv = *reinterpret_cast<const float2*>(xs + row * ROWW + col);
                        float x0 = p.alpha * mv.x, x1 = p.alpha * mv.y;
                        if (p.add_identity && row == col) x0 += 1.0f;
                        if (p.add_identity && row == col + 1) x1 += 1.0f;
                        part = fmaf(D[nt][2 * h8], x0, fmaf(D[nt][2 * h8 + 1], x1, part));
                    }
                part = warp_sum(part);
                if (lane == 0) sm.c.red2[warp] = part;
            }
        }
        // ---- the determinant scale and the inverse's series terms; its barrier
        // (or the one in its place) also publishes the parts of <dX, Xr> and
        // ends every warp's reads of S and G ----
        float Y[8][4];
        Series sr;
        sr.ok = !detnorm;
        sr.inv_ok = !detnorm;
        sr.cm1 = 0.0f;
        if (series) sr = det_series<true>(sm.c, xs, p.alpha, warp, lane, Y);
        else if (out_tok) __syncthreads();
        // ---- where the series does not serve: the pivoted elimination ----
        const bool elim = detnorm && (!sr.ok || (out_tok && !sr.inv_ok));     // uniform over the CTA
        float cm1 = sr.cm1;
        bool good = true;
        if (elim) {
            const double ld = pivoted_logdet(sm.c, xs, out_tok ? sm.s : nullptr, p.alpha, p.add_identity);
            reload_slice(xs, x + base + tau * tok);
            if (!sr.ok) {
                good = isfinite(ld);
                cm1 = (float)expm1(-ld / N);
            }
        }
        const Scale sc = finish_scale(p, detnorm, cm1, good, status);
        // ---- the embedding gradient ----
        if (out_tok) {
            float* out = dx + base + tau * tok;
            if (!detnorm) {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8)
                        *reinterpret_cast<float2*>(out + (r0 + g + 8 * h8) * N + 8 * nt + 2 * q) =
                            make_float2(p.alpha * D[nt][2 * h8], p.alpha * D[nt][2 * h8 + 1]);
            } else {
                const float s = ((sm.c.red2[0] + sm.c.red2[1]) + (sm.c.red2[2] + sm.c.red2[3])) * (1.0f / N);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                        float o[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            // Xr^-T at (row, col + e)
                            float zi;
                            if (elim) {
                                zi = sm.s[(col + e) * ROWW + row];
                            } else {
                                zi = fmaf(-p.alpha, xs[(col + e) * ROWW + row], Y[nt][2 * h8 + e]);
                                if (row == col + e) zi += 1.0f;
                            }
                            o[e] = sc.c == 0.0f ? 0.0f : sc.ca * fmaf(-s, zi, D[nt][2 * h8 + e]);
                        }
                        *reinterpret_cast<float2*>(out + row * N + col) = make_float2(o[0], o[1]);
                    }
            }
            if (elim) __syncthreads();               // the inverse has been read: the buffer takes S again
            if (tau > t0) issue_state(sm.s, p, S_fwd, S0, base, tok, bh, tau - 1);
        }
        // ---- G_{tau-1} = dS_{tau-1} + G X_tau^T, or dS0 = G X_1^T ----
        if (tau > t0 || (tau == 0 && dS0 != nullptr)) {
            float A[8][4];
            zero(A);
#pragma unroll
            for (int kt = 0; kt < 8; ++kt) {
                // this warp's rows of G, the contraction permuted as for frag_mt
                uint32_t a[4];
                const float2 u0 = *reinterpret_cast<const float2*>(sm.g + (r0 + g) * ROWW + 8 * kt + 2 * q);
                const float2 u1 = *reinterpret_cast<const float2*>(sm.g + (r0 + g + 8) * ROWW + 8 * kt + 2 * q);
                a[0] = to_tf32(u0.x);
                a[1] = to_tf32(u1.x);
                a[2] = to_tf32(u0.y);
                a[3] = to_tf32(u1.y);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    uint32_t b0, b1;
                    frag_mt(xs, kt, nt, g, q, b0, b1);
                    mma_tf32(A[nt], a, b0, b1);
                }
            }
            // each lane's A fragments were its own accumulator positions of G,
            // so it overwrites only what it alone has read
            const bool to_g = tau > t0;
            float* dst = to_g ? sm.g : dS0 + bh * NN;
            const int ld = to_g ? ROWW : N;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const int row = r0 + g + 8 * h8, col = 8 * nt + 2 * q;
                    const float2 go = *reinterpret_cast<const float2*>(sm.g + row * ROWW + col);
                    const float y0 = dsr[nt][h8].x + (go.x + fmaf(sc.ca, A[nt][2 * h8], sc.dv * go.x));
                    const float y1 = dsr[nt][h8].y + (go.y + fmaf(sc.ca, A[nt][2 * h8 + 1], sc.dv * go.y));
                    *reinterpret_cast<float2*>(dst + row * ld + col) = make_float2(y0, y1);
                }
        }
    }
    cp_wait_all();
}

}  // namespace

// tf32 arithmetic explicitly asked for, fp32 embeddings, reshape or
// determinant-corrected construction.
bool supports_backward(const KParams& p)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_F32 && p.math == MRU_MATH_TF32 &&
           (p.mode == MRU_MODE_DETNORM || p.mode == MRU_MODE_RESHAPE);
}

cudaError_t launch_bwd_local(const KParams& p, const float* x, const float* dS, float* gloc, float* Wq,
                             uint32_t* status, cudaStream_t s)
{
    const int64_t chains = p.B * p.H * p.K;
    if (chains == 0) return cudaSuccess;
    const size_t sm = sizeof(LocalSmem);
    cudaError_t e = cudaFuncSetAttribute(k64b_local, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k64b_local<<<(unsigned)chains, THREADS, sm, s>>>(p, x, dS, gloc, Wq, status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_apply(const KParams& p, const float* x, const float* S0, const float* S_fwd, const float* dS,
                             const float* Gin, float* dx, float* dS0, uint32_t* status, cudaStream_t s)
{
    const int64_t chains = p.B * p.H * p.K;
    if (chains == 0) return cudaSuccess;
    const size_t sm = sizeof(ApplySmem);
    cudaError_t e = cudaFuncSetAttribute(k64b_apply, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k64b_apply<<<(unsigned)chains, THREADS, sm, s>>>(p, x, S0, S_fwd, dS, Gin, dx, dS0, status);
    return cudaGetLastError();
}

}  // namespace n64
}  // namespace mru
