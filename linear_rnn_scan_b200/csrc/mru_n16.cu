// mru_n16.cu -- n = 16 scan kernels on the tensor cores (fp32 embeddings,
// reshape and determinant-corrected modes), two passes over the embeddings:
//
//  * reduce pass   one warp per chain (b, h, chunk of C = 8m tokens); warps
//                  never wait for each other.  Per pass of 8 tokens the warp
//                  copies the 8 token-head slices to its shared memory
//                  (cp.async, rows padded to 20 words), factorises the 8
//                  matrices at once with 4 lanes per token (lane r owns rows
//                  r, r+4, r+8, r+12 in registers; the pivot row is broadcast
//                  by shuffles inside the 4-lane group), records the token's
//                  scalars (c alpha, diagonal of F) and advances the chunk
//                  product Q_t = Q_{t-1} + (F_t + Q_{t-1} F_t) with mma.sync
//                  m16n8k8 tf32 in split precision.  The state stays in the
//                  accumulator registers from token to token: the contraction
//                  index of the next product is permuted so that the
//                  accumulator fragment of column tile j is exactly the A
//                  fragment of k-tile j.  Only the chunk total is written.
//  * (the fp64 scan of chunk totals, mru_carry.cu)
//  * apply pass    one warp per chain: forms the chunk's exact carry from the
//                  carry scan (fp64), then runs the chain again from it,
//                  S_t = S_{t-1} + S_{t-1} F_t, and writes every S_t.  No local
//                  prefix ever goes to memory: per token·head the path moves
//                  x twice and S once.
//
// Split-tf32 ("3xTF32", after Ootomo and Yokota, 2022): x = hi + lo with hi
// the top 19 bits of x (sign, exponent, 10 mantissa bits) and lo = x - hi
// exact in fp32; a b ~ a_lo b_hi + a_hi b_lo + a_hi b_hi.
#include <string.h>

#include "mru_internal.cuh"

namespace mru {
namespace n16 {
namespace {

constexpr int N = 16;
constexpr int NN = N * N;
constexpr int ROWW = 20;            // padded shared-memory row stride, in words
constexpr int SLICE = N * ROWW;     // one token-head slice in shared memory
constexpr int SUB = kSub;           // tokens per pass
constexpr int WARPS = 8;            // chains per CTA
constexpr int THREADS = 32 * WARPS;

struct WarpSmem {
    float x[SUB][SLICE];            // 10,240 bytes
    float2 cd[SUB];                 // (c * alpha, diagonal term of F) per token
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

__device__ __forceinline__ void mma_3xtf32(float (&acc)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                           const uint32_t (&bh)[2], const uint32_t (&bl)[2])
{
    mma_tf32(acc, al, bh);
    mma_tf32(acc, ah, bl);
    mma_tf32(acc, ah, bh);
}

// log|det(W)| of one 16 x 16 matrix held by a group of 4 lanes (lane r owns
// rows r, r+4, r+8, r+12 in e[0..3][0..15]).  near_identity: W = I + e,
// eliminated on e alone without pivoting, |det| = prod |1 + delta_k| in fp64;
// returns false when a pivot |1 + delta_k| < 0.5.  Otherwise W = e with
// partial pivoting, log|det| summed in fp64.  Every lane of the warp must
// call it with the same near_identity (the shuffles span the warp).
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
            // swap rows k and bi (row i lives in lane i & 3, slot i >> 2);
            // unconditional (a no-op when bi == k) to keep the warp converged
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
        float prow[N];
#pragma unroll
        for (int j = k; j < N; ++j) prow[j] = __shfl_sync(full, e[kr][j], owner, 4);
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
        const float rk = (pk != 0.0f) ? __frcp_rn(pk) : 0.0f;
#pragma unroll
        for (int lr = 0; lr < 4; ++lr) {
            if (4 * lr + 3 <= k) continue;        // no row of this slot is below k
            const int i = 4 * lr + r;
            if (i > k) {
                const float l = e[lr][k] * rk;
#pragma unroll
                for (int j = k + 1; j < N; ++j) e[lr][j] = fmaf(-l, prow[j], e[lr][j]);
            }
        }
    }
    logabs = near_identity ? log(fabs(prod)) : lsum;
    return ok;
}

// Copies the slices of tokens [t0, t0 + nt) of one (b, h) into the warp's
// shared memory (16-byte granules, rows padded to ROWW words).
__device__ __forceinline__ void load_pass(WarpSmem& ws, const float* xb, int64_t tok, int64_t t0, int nt, int lane)
{
#pragma unroll
    for (int i = 0; i < SUB * 64 / 32; ++i) {
        const int gi = lane + 32 * i;
        const int j = gi >> 6, q16 = gi & 63, row = q16 >> 2, col4 = q16 & 3;
        if (j < nt) cp_async16(&ws.x[j][row * ROWW + col4 * 4], xb + (t0 + j) * tok + row * N + col4 * 4);
    }
    cp_async_wait_all();
    __syncwarp();
}

// The per-token scalars of F = ca * M + dv * I for the 8 tokens of a pass:
// 4-lane LU groups for the determinant-corrected mode.  Lane r == 0 of each
// group writes ws.cd[group].
__device__ __forceinline__ void pass_scalars(const KParams& p, WarpSmem& ws, int nt, int lane, uint32_t* status)
{
    const int grp = lane >> 2, r = lane & 3;
    const bool live = grp < nt;
    float ca = p.alpha, dv = p.add_identity ? 0.0f : -1.0f;
    if (p.mode == MRU_MODE_DETNORM) {
        float e[4][N];
        const float* xs = ws.x[grp];
#pragma unroll
        for (int lr = 0; lr < 4; ++lr) {
            const float4* row4 = reinterpret_cast<const float4*>(xs + (4 * lr + r) * ROWW);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 v = live ? row4[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
                e[lr][4 * c4 + 0] = p.alpha * v.x;
                e[lr][4 * c4 + 1] = p.alpha * v.y;
                e[lr][4 * c4 + 2] = p.alpha * v.z;
                e[lr][4 * c4 + 3] = p.alpha * v.w;
            }
        }
        double ld = 0.0;
        bool singular = false, ok = true;
        if (p.add_identity) ok = group_logabsdet(e, r, true, ld, singular);
        if (__any_sync(0xffffffffu, !p.add_identity || !ok)) {
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
        const float c = (float)(1.0 + cm1d);
        if (singular || !isfinite(ld) || !isfinite(c) || c == 0.0f) {
            if (live && r == 0) atomicOr(status, STATUS_SINGULAR);
            ca = 0.0f;                       // output unspecified; keep X = I
            dv = 0.0f;
        } else {
            ca = c * p.alpha;
            dv = p.add_identity ? (float)cm1d : -1.0f;
        }
    }
    if (r == 0) ws.cd[grp] = make_float2(ca, dv);
    __syncwarp();
}

// B fragments (split) of F = ca * M + dv * I for one token, with the
// contraction index permuted (slot q <-> row 8kt + 2q, slot q + 4 <-> row
// 8kt + 2q + 1), and F at this lane's accumulator positions.
struct FragF {
    uint32_t bh[2][2][2], bl[2][2][2];
    float fd[2][4];
};

__device__ __forceinline__ void make_frag_f(const float* xs, float ca, float d0, float d1, int g, int q, FragF& f,
                                            bool want_fd)
{
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float* base = xs + (8 * kt + 2 * q) * ROWW + 8 * nt + g;
            const float v0 = fmaf(ca, base[0], kt == nt ? d0 : 0.0f);
            const float v1 = fmaf(ca, base[ROWW], kt == nt ? d1 : 0.0f);
            split_tf32(v0, f.bh[kt][nt][0], f.bl[kt][nt][0]);
            split_tf32(v1, f.bh[kt][nt][1], f.bl[kt][nt][1]);
        }
    if (want_fd) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const float2 xv = *reinterpret_cast<const float2*>(xs + (g + 8 * h8) * ROWW + 8 * nt + 2 * q);
                f.fd[nt][2 * h8 + 0] = fmaf(ca, xv.x, h8 == nt ? d0 : 0.0f);
                f.fd[nt][2 * h8 + 1] = fmaf(ca, xv.y, h8 == nt ? d1 : 0.0f);
            }
    }
}

// acc = A F with A the 16 x 16 state held in accumulator layout (Ad).
__device__ __forceinline__ void chain_product(const float (&Ad)[2][4], const FragF& f, float (&acc)[2][4])
{
    uint32_t ah[2][4], al[2][4];
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
        split_tf32(Ad[kt][0], ah[kt][0], al[kt][0]);
        split_tf32(Ad[kt][2], ah[kt][1], al[kt][1]);
        split_tf32(Ad[kt][1], ah[kt][2], al[kt][2]);
        split_tf32(Ad[kt][3], ah[kt][3], al[kt][3]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) mma_3xtf32(acc[nt], ah[kt], al[kt], f.bh[kt][nt], f.bl[kt][nt]);
    }
}

__device__ __forceinline__ void store_d(float* out, const float (&Ad)[2][4], int g, int q)
{
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8)
            *reinterpret_cast<float2*>(out + (g + 8 * h8) * N + 8 * nt + 2 * q) =
                make_float2(Ad[nt][2 * h8], Ad[nt][2 * h8 + 1]);
}

// chain id -> (b, k, h), h fastest: a CTA's chains are neighbouring heads of
// one token range (their slices are contiguous in memory).
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

// ---- chain bodies, shared by the two-pass kernels and the fused kernel ----

// The reduce chain of one warp over tokens [tbeg, tend): per-token scalars to
// cdb[t * H] and the chunk total (split form) left in Qd.
__device__ __forceinline__ void reduce_chain(const KParams& p, WarpSmem& ws, const float* xb, int64_t tok,
                                             float2* cdb, int64_t tbeg, int64_t tend, int lane, uint32_t* status,
                                             float (&Qd)[2][4])
{
    const int g = lane >> 2, q = lane & 3;
    const float m0 = (g == 2 * q) ? 1.0f : 0.0f;         // diagonal positions of this lane's fragments
    const float m1 = (g == 2 * q + 1) ? 1.0f : 0.0f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) Qd[nt][i] = 0.0f;
    for (int64_t t0 = tbeg; t0 < tend; t0 += SUB) {
        const int nt_pass = (tend - t0 < SUB) ? (int)(tend - t0) : SUB;
        load_pass(ws, xb, tok, t0, nt_pass, lane);
        pass_scalars(p, ws, nt_pass, lane, status);
        if (lane < nt_pass) cdb[(t0 + lane) * p.H] = ws.cd[lane];
        for (int j = 0; j < nt_pass; ++j) {
            const float2 cdj = ws.cd[j];
            FragF f;
            make_frag_f(ws.x[j], cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, f, true);
            float acc[2][4];
            chain_product(Qd, f, acc);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) Qd[nt][i] += f.fd[nt][i] + acc[nt][i];
        }
        __syncwarp();
    }
}

// The chain's carry C = E (I + R) in fp64 (R may be null: C = E), rounded to
// fp32, into accumulator layout Sd.  Uses the warp's x buffer as scratch.
__device__ __forceinline__ void form_carry(WarpSmem& ws, const double* E, const float* R, int lane,
                                           float (&Sd)[2][4])
{
    double* sE = reinterpret_cast<double*>(&ws.x[0][0]);      // 2 KB
    float* sC = reinterpret_cast<float*>(&ws.x[2][0]);        // 1 KB
    for (int e = lane; e < NN; e += 32) sE[e] = E[e];
    __syncwarp();
    const int r0 = (lane >> 2) * 2, c0 = (lane & 3) * 4;
    double acc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) acc[i][cc] = 0.0;
    if (R) {
#pragma unroll 4
        for (int kk = 0; kk < N; ++kk) {
            const double a0 = sE[r0 * N + kk], a1 = sE[(r0 + 1) * N + kk];
            const float4 rv = *reinterpret_cast<const float4*>(R + kk * N + c0);
            const double bv[4] = {(double)rv.x, (double)rv.y, (double)rv.z, (double)rv.w};
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                acc[0][cc] = fma(a0, bv[cc], acc[0][cc]);
                acc[1][cc] = fma(a1, bv[cc], acc[1][cc]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
            sC[(r0 + i) * N + c0 + cc] = (float)(sE[(r0 + i) * N + c0 + cc] + acc[i][cc]);
    __syncwarp();
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const float2 v = *reinterpret_cast<const float2*>(sC + (g + 8 * h8) * N + 8 * nt + 2 * q);
            Sd[nt][2 * h8] = v.x;
            Sd[nt][2 * h8 + 1] = v.y;
        }
    __syncwarp();
}

// The apply chain of one warp: S_t = S_{t-1} + S_{t-1} F_t from Sd, every
// S_t written to ob + t * tok.
__device__ __forceinline__ void apply_chain(WarpSmem& ws, const float* xb, float* ob, int64_t tok, int64_t H,
                                            const float2* cdb, int64_t tbeg, int64_t tend, int lane,
                                            float (&Sd)[2][4])
{
    const int g = lane >> 2, q = lane & 3;
    const float m0 = (g == 2 * q) ? 1.0f : 0.0f;
    const float m1 = (g == 2 * q + 1) ? 1.0f : 0.0f;
    for (int64_t t0 = tbeg; t0 < tend; t0 += SUB) {
        const int nt_pass = (tend - t0 < SUB) ? (int)(tend - t0) : SUB;
        // the pass's per-token scalars travel with the slice copies (they
        // would otherwise be a dependent global load per token)
        if (lane < nt_pass) ws.cd[lane] = cdb[(t0 + lane) * H];
        load_pass(ws, xb, tok, t0, nt_pass, lane);
        for (int j = 0; j < nt_pass; ++j) {
            const float2 cdj = ws.cd[j];
            FragF f;
            make_frag_f(ws.x[j], cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, f, false);
            float acc[2][4];
            chain_product(Sd, f, acc);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) Sd[nt][i] += acc[nt][i];
            store_d(ob + (t0 + j) * tok, Sd, g, q);
        }
        __syncwarp();
    }
}

// Reduce pass: chunk totals (split form) and per-token scalars.
__global__ void __launch_bounds__(THREADS, 2)
k16_reduce(KParams p, const float* __restrict__ x, float* __restrict__ totals, float2* __restrict__ cd_out,
           uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem_raw)[warp];
    const int64_t chain = (int64_t)blockIdx.x * WARPS + warp;
    if (chain >= p.B * p.H * p.K) return;
    const ChainIx c = chain_ix(p, chain);
    const int64_t tok = p.H * NN;
    const float* xb = x + (c.b * p.L * p.H + c.h) * NN;
    float2* cdb = cd_out + c.b * p.L * p.H + c.h;
    float Qd[2][4];
    reduce_chain(p, ws, xb, tok, cdb, c.tbeg, c.tend, lane, status, Qd);
    store_d(totals + ((c.b * p.H + c.h) * p.K + c.k) * NN, Qd, lane >> 2, lane & 3);
}

// Apply pass: the chunk's carry C = E1 (I + R0[k-1]) in fp64, then
// S_t = S_{t-1} + S_{t-1} F_t from S = C, every S_t written.
__global__ void __launch_bounds__(THREADS, 2)
k16_apply(KParams p, const float* __restrict__ x, const float2* __restrict__ cd_in, const float* __restrict__ R0,
          const double* __restrict__ E1, int G, float* __restrict__ S_out)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem_raw)[warp];
    const int64_t chain = (int64_t)blockIdx.x * WARPS + warp;
    if (chain >= p.B * p.H * p.K) return;
    const ChainIx c = chain_ix(p, chain);
    const int64_t seq = c.b * p.H + c.h;
    const int64_t n1 = (p.K + G - 1) / G;
    float Sd[2][4];
    form_carry(ws, E1 + (seq * n1 + c.k / G) * NN, (c.k % G) ? R0 + (seq * p.K + c.k - 1) * NN : nullptr, lane, Sd);
    const int64_t tok = p.H * NN;
    apply_chain(ws, x + (c.b * p.L * p.H + c.h) * NN, S_out + (c.b * p.L * p.H + c.h) * NN, tok, p.H,
                cd_in + c.b * p.L * p.H + c.h, c.tbeg, c.tend, lane, Sd);
}

// ---- fused persistent kernel --------------------------------------------
//
// One launch runs the whole scan as a dataflow of work items over windows of
// Kw chunks (all sequences), taken in ticket order from a global counter:
//     R(0) .. R(lag-1), then per window w:  R(w+lag), S1(w), S2(w), A(w)
//   R(w)   reduce chains of window w: chunk totals + per-token scalars
//   S1(w)  per (sequence, group of G chunks): fp64 inclusive local prefixes
//          R0 (kept fp32) and the group total Tot (fp64)
//   S2(w)  per sequence: exclusive group carries E1 from the running carry
//          (fp64), which it hands on to S2(w+1)
//   A(w)   apply chains of window w from their exact carries, S_t written
// An item only waits for items with smaller tickets (S1(w) for all R(w),
// S2(w) for all S1(w) and S2(w-1), A(w) for S2(w)); those are held by CTAs
// that are running, so the waits end.  Each wait is bounded: past the limit
// the kernel records STATUS_TIMEOUT, raises the abort flag and returns.
// Windows are sized so that the embeddings of the lag + 1 windows in flight
// stay in L2, where the apply pass reads them the second time.

constexpr unsigned kSpinLimit = 4u << 20;     // x up to ~1 us of back-off: a few seconds

struct FusedCfg {
    int G;              // chunks per group
    int Kw;             // chunks per window (multiple of G)
    int lag;            // windows the reduce items run ahead
    int64_t NW;         // windows
    int64_t nR, nS1, nS2, nA;
    int64_t total;      // tickets
    int64_t NG;         // groups per sequence
};

struct FusedBufs {
    unsigned* ticket;
    unsigned* abort_flag;
    unsigned* cntR;     // [NW]
    unsigned* cntS1;    // [NW]
    unsigned* cntS2;    // [NW]
    float* totals;      // [seq][K]
    float2* cd;         // [B][L][H]
    float* R0;          // [seq][K]
    double* Tot;        // [seq][NG]
    double* E1;         // [seq][NG]
    double* cstate;     // [seq]
    uint32_t* status;
};

__device__ __forceinline__ unsigned ld_volatile(const unsigned* p)
{
    return *reinterpret_cast<const volatile unsigned*>(p);
}

// Called by thread 0 only.  True once *ctr >= target; false on timeout or
// when another CTA has aborted.
__device__ bool wait_geq(const unsigned* ctr, unsigned target, const FusedBufs& fb)
{
    unsigned ns = 32;
    for (unsigned spins = 0;; ++spins) {
        if (ld_volatile(ctr) >= target) {
            __threadfence();
            return true;
        }
        if (ld_volatile(fb.abort_flag)) return false;
        if (spins >= kSpinLimit) {
            atomicOr(fb.status, STATUS_TIMEOUT);
            atomicExch(fb.abort_flag, 1u);
            return false;
        }
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
    }
}

// C = A B for 16 x 16 fp64 matrices in shared memory; lane owns a 2 x 4 block.
__device__ __forceinline__ void warp_gemm16_f64(const double* A, const double* B, int lane, double (&acc)[2][4])
{
    const int r0 = (lane >> 2) * 2, c0 = (lane & 3) * 4;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = 0.0;
#pragma unroll 4
    for (int k = 0; k < N; ++k) {
        const double a0 = A[r0 * N + k], a1 = A[(r0 + 1) * N + k];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const double b = B[k * N + c0 + c];
            acc[0][c] = fma(a0, b, acc[0][c]);
            acc[1][c] = fma(a1, b, acc[1][c]);
        }
    }
}

// chain index inside window w -> global chain coordinates (h fastest, then
// the chunk within the window, then b); false when outside the problem.
__device__ __forceinline__ bool window_chain(const KParams& p, const FusedCfg& fc, int64_t w, int64_t ci, ChainIx& c)
{
    if (ci >= p.B * (int64_t)fc.Kw * p.H) return false;
    c.h = ci % p.H;
    const int64_t kk = (ci / p.H) % fc.Kw;
    c.b = ci / (p.H * (int64_t)fc.Kw);
    c.k = w * fc.Kw + kk;
    if (c.k >= p.K) return false;
    c.tbeg = c.k * p.chunk;
    c.tend = (c.tbeg + p.chunk < p.L) ? c.tbeg + p.chunk : p.L;
    return true;
}

__global__ void __launch_bounds__(THREADS, 2)
k16_fused(KParams p, FusedCfg fc, FusedBufs fb, const float* __restrict__ x, const float* __restrict__ S0,
          float* __restrict__ S_out)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int64_t s_ticket;
    __shared__ int s_go;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(smem_raw)[warp];
    const int64_t tok = p.H * NN;
    const int64_t nseq = p.B * p.H;
    const int gpw = fc.Kw / fc.G;                    // groups per window

    for (;;) {
        if (tid == 0) s_ticket = ld_volatile(fb.abort_flag) ? fc.total : (int64_t)atomicAdd(fb.ticket, 1u);
        __syncthreads();
        const int64_t t = s_ticket;
        __syncthreads();
        if (t >= fc.total) return;

        int kind;                                    // 0 R, 1 S1, 2 S2, 3 A
        int64_t w, idx;
        if (t < fc.lag * fc.nR) {
            kind = 0; w = t / fc.nR; idx = t % fc.nR;
        } else {
            const int64_t bs = fc.nR + fc.nS1 + fc.nS2 + fc.nA;
            const int64_t u = t - fc.lag * fc.nR;
            w = u / bs;
            int64_t r = u % bs;
            if (r < fc.nR) { kind = 0; w += fc.lag; idx = r; }
            else if ((r -= fc.nR) < fc.nS1) { kind = 1; idx = r; }
            else if ((r -= fc.nS1) < fc.nS2) { kind = 2; idx = r; }
            else { kind = 3; idx = r - fc.nS2; }
        }
        if (kind == 0 && w >= fc.NW) continue;       // past the last window: nothing to do

        // ---- wait for this item's inputs ----
        if (tid == 0) {
            bool ok = true;
            if (kind == 1) ok = wait_geq(fb.cntR + w, (unsigned)fc.nR, fb);
            if (kind == 2) {
                ok = wait_geq(fb.cntS1 + w, (unsigned)fc.nS1, fb);
                if (ok && w > 0) ok = wait_geq(fb.cntS2 + w - 1, (unsigned)fc.nS2, fb);
            }
            if (kind == 3) ok = wait_geq(fb.cntS2 + w, (unsigned)fc.nS2, fb);
            s_go = ok;
        }
        __syncthreads();
        if (!s_go) return;

        if (kind == 0) {
            ChainIx c;
            if (window_chain(p, fc, w, idx * WARPS + warp, c)) {
                float Qd[2][4];
                reduce_chain(p, ws, x + (c.b * p.L * p.H + c.h) * NN, tok, fb.cd + c.b * p.L * p.H + c.h,
                             c.tbeg, c.tend, lane, fb.status, Qd);
                store_d(fb.totals + ((c.b * p.H + c.h) * p.K + c.k) * NN, Qd, lane >> 2, lane & 3);
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) atomicAdd(fb.cntR + w, 1u);
        } else if (kind == 1) {
            const int64_t gi = idx * WARPS + warp;
            const int64_t seq = gi / gpw;
            const int64_t gg = w * gpw + gi % gpw;
            if (seq < nseq && gg * fc.G < p.K) {
                double* sR = reinterpret_cast<double*>(&ws.x[0][0]);
                double* sT = sR + NN;
                const int r0 = (lane >> 2) * 2, c0 = (lane & 3) * 4;
                for (int e = lane; e < NN; e += 32) sR[e] = 0.0;
                const int64_t k1 = (gg + 1) * fc.G < p.K ? (gg + 1) * fc.G : p.K;
                for (int64_t k = gg * fc.G; k < k1; ++k) {
                    const float* tk = fb.totals + (seq * p.K + k) * NN;
                    for (int e = lane; e < NN; e += 32) sT[e] = (double)tk[e];
                    __syncwarp();
                    double acc[2][4];
                    warp_gemm16_f64(sR, sT, lane, acc);
                    __syncwarp();
                    float* rk = fb.R0 + (seq * p.K + k) * NN;
#pragma unroll
                    for (int i = 0; i < 2; ++i)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            const int e = (r0 + i) * N + c0 + cc;
                            const double v = sR[e] + (sT[e] + acc[i][cc]);
                            sR[e] = v;
                            rk[e] = (float)v;
                        }
                    __syncwarp();
                }
                double* tot = fb.Tot + (seq * fc.NG + gg) * NN;
                for (int e = lane; e < NN; e += 32) tot[e] = sR[e];
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) atomicAdd(fb.cntS1 + w, 1u);
        } else if (kind == 2) {
            const int64_t seq = idx * WARPS + warp;
            if (seq < nseq) {
                double* sG = reinterpret_cast<double*>(&ws.x[0][0]);
                double* sT = sG + NN;
                const int r0 = (lane >> 2) * 2, c0 = (lane & 3) * 4;
                for (int e = lane; e < NN; e += 32)
                    sG[e] = (w > 0) ? fb.cstate[seq * NN + e]
                                    : (S0 ? (double)S0[seq * NN + e] : ((e / N) == (e % N) ? 1.0 : 0.0));
                __syncwarp();
                for (int gw = 0; gw < gpw; ++gw) {
                    const int64_t gg = w * gpw + gw;
                    if (gg >= fc.NG) break;
                    double* e1 = fb.E1 + (seq * fc.NG + gg) * NN;
                    const double* tg = fb.Tot + (seq * fc.NG + gg) * NN;
                    for (int e = lane; e < NN; e += 32) {
                        e1[e] = sG[e];
                        sT[e] = tg[e];
                    }
                    __syncwarp();
                    double acc[2][4];
                    warp_gemm16_f64(sG, sT, lane, acc);
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 2; ++i)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) sG[(r0 + i) * N + c0 + cc] += acc[i][cc];
                    __syncwarp();
                }
                for (int e = lane; e < NN; e += 32) fb.cstate[seq * NN + e] = sG[e];
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) atomicAdd(fb.cntS2 + w, 1u);
        } else {
            ChainIx c;
            if (window_chain(p, fc, w, idx * WARPS + warp, c)) {
                const int64_t seq = c.b * p.H + c.h;
                float Sd[2][4];
                form_carry(ws, fb.E1 + (seq * fc.NG + c.k / fc.G) * NN,
                           (c.k % fc.G) ? fb.R0 + (seq * p.K + c.k - 1) * NN : nullptr, lane, Sd);
                apply_chain(ws, x + (c.b * p.L * p.H + c.h) * NN, S_out + (c.b * p.L * p.H + c.h) * NN, tok, p.H,
                            fb.cd + c.b * p.L * p.H + c.h, c.tbeg, c.tend, lane, Sd);
            }
            __syncthreads();
        }
    }
}

}  // namespace

bool supports(const KParams& p, bool readout)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_F32 && !readout &&
           (p.mode == MRU_MODE_RESHAPE || p.mode == MRU_MODE_DETNORM) &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_TF32X3) && p.chunk > 0 && p.chunk % SUB == 0;
}

// Chunk length: 8 tokens per pass, m passes per chain, m a power of two that
// keeps at least 16384 chains (about 7 waves of 16 warps per SM) when the
// workload allows, so that long sequences get long chunks (few chunk totals).
int32_t preferred_chunk(int64_t token_heads)
{
    int32_t m = 1;
    while (m < 16 && token_heads / ((int64_t)SUB * 2 * m) >= 16384) m *= 2;
    return SUB * m;
}

cudaError_t launch_reduce(const KParams& p, const float* x, float* totals, float2* cd, uint32_t* status,
                          cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    const unsigned grid = (unsigned)((nchains + WARPS - 1) / WARPS);
    const size_t sm = sizeof(WarpSmem) * WARPS;
    cudaError_t e = cudaFuncSetAttribute(k16_reduce, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k16_reduce<<<grid, THREADS, sm, s>>>(p, x, totals, cd, status);
    return cudaGetLastError();
}

cudaError_t launch_apply(const KParams& p, const float* x, const float2* cd, const carry::Plan& pl,
                         const char* ws, float* S_out, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    const unsigned grid = (unsigned)((nchains + WARPS - 1) / WARPS);
    const size_t sm = sizeof(WarpSmem) * WARPS;
    cudaError_t e = cudaFuncSetAttribute(k16_apply, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k16_apply<<<grid, THREADS, sm, s>>>(p, x, cd, reinterpret_cast<const float*>(ws + pl.R[0]),
                                        reinterpret_cast<const double*>(ws + pl.E[1]), pl.G, S_out);
    return cudaGetLastError();
}

// Layout of the fused kernel's workspace from byte offset `off` (the first
// bytes, counters and flags, must be zeroed before every launch).
FusedLayout fused_layout(const KParams& p, size_t off)
{
    FusedLayout L;
    memset(&L, 0, sizeof L);
    const int64_t nseq = p.B * p.H;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) / 256 * 256;
        return o;
    };
    L.G = 16;
    const int64_t unit = nseq * (int64_t)p.chunk * L.G * NN * (int64_t)sizeof(float);  // x bytes per group of chunks
    int64_t groups = (16ll << 20) / (unit > 0 ? unit : 1);
    if (groups < 1) groups = 1;
    if (groups > 64) groups = 64;
    L.Kw = (int)(groups * L.G);
    L.NW = p.K > 0 ? (p.K + L.Kw - 1) / L.Kw : 0;
    L.NG = (p.K + L.G - 1) / L.G;
    L.counters = take(sizeof(unsigned) * (2 + 3 * (size_t)L.NW));
    L.counters_bytes = sizeof(unsigned) * (2 + 3 * (size_t)L.NW);
    L.totals = take(sizeof(float) * nseq * p.K * NN);
    L.cd = take(sizeof(float2) * nseq * p.L);
    L.R0 = take(sizeof(float) * nseq * p.K * NN);
    L.Tot = take(sizeof(double) * nseq * L.NG * NN);
    L.E1 = take(sizeof(double) * nseq * L.NG * NN);
    L.cstate = take(sizeof(double) * nseq * NN);
    L.end = off;
    return L;
}

cudaError_t launch_fused(const KParams& p, const FusedLayout& L, char* ws, uint32_t* status, const float* x,
                         const float* S0, float* S_out, cudaStream_t s)
{
    const int64_t nseq = p.B * p.H;
    if (nseq * p.K == 0) return cudaSuccess;
    FusedCfg fc;
    fc.G = L.G;
    fc.Kw = L.Kw;
    fc.lag = 2;
    fc.NW = L.NW;
    fc.NG = L.NG;
    const int64_t chains_w = p.B * (int64_t)L.Kw * p.H;
    fc.nR = (chains_w + WARPS - 1) / WARPS;
    fc.nA = fc.nR;
    fc.nS1 = (nseq * (L.Kw / L.G) + WARPS - 1) / WARPS;
    fc.nS2 = (nseq + WARPS - 1) / WARPS;
    fc.total = fc.lag * fc.nR + fc.NW * (fc.nR + fc.nS1 + fc.nS2 + fc.nA);
    FusedBufs fb;
    unsigned* ctr = reinterpret_cast<unsigned*>(ws + L.counters);
    fb.ticket = ctr;
    fb.abort_flag = ctr + 1;
    fb.cntR = ctr + 2;
    fb.cntS1 = ctr + 2 + L.NW;
    fb.cntS2 = ctr + 2 + 2 * L.NW;
    fb.totals = reinterpret_cast<float*>(ws + L.totals);
    fb.cd = reinterpret_cast<float2*>(ws + L.cd);
    fb.R0 = reinterpret_cast<float*>(ws + L.R0);
    fb.Tot = reinterpret_cast<double*>(ws + L.Tot);
    fb.E1 = reinterpret_cast<double*>(ws + L.E1);
    fb.cstate = reinterpret_cast<double*>(ws + L.cstate);
    fb.status = status;
    cudaError_t e = cudaMemsetAsync(ws + L.counters, 0, L.counters_bytes, s);
    if (e != cudaSuccess) return e;
    const size_t sm = sizeof(WarpSmem) * WARPS;
    e = cudaFuncSetAttribute(k16_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k16_fused, THREADS, sm)) != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = (int64_t)sms * per_sm;
    if (grid > fc.total) grid = fc.total;
    k16_fused<<<(unsigned)grid, THREADS, sm, s>>>(p, fc, fb, x, S0, S_out);
    return cudaGetLastError();
}

}  // namespace n16
}  // namespace mru
