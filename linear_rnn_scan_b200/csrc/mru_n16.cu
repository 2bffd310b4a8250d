// mru_n16.cu -- n = 16 scan kernels on the tensor cores (fp32 embeddings,
// reshape and determinant-corrected modes): three launches, two passes over
// the embeddings; and the backward's two passes (at the end of the file).
//
// Both passes run persistent warps: warp w of W takes the chains (b, h,
// chunk of C tokens) w, w + W, w + 2W, ... (a CTA's warps hold neighbouring
// heads of one token range, whose slices are contiguous) and streams their
// token-head slices through a cp.async pipeline in its own shared memory,
// across chain boundaries; while it computes on one stage the next ones are
// in flight.  Warps never wait for each other.
//
//  * reduce pass   the chunk product Q_t = Q_{t-1} + (F_t + Q_{t-1} F_t)
//                  (P = I + Q, X = I + F) on mma.sync m16n8k8 tf32 in split
//                  precision; the state stays in the accumulator registers
//                  from token to token (the contraction index of the next
//                  product is permuted so that the accumulator fragment of
//                  column tile j is exactly the A fragment of k-tile j).  In
//                  the determinant-corrected mode with the identity added the
//                  chain runs on the uncorrected matrices: the determinant is
//                  multiplicative, so the product of the corrected matrices
//                  is gamma P~ with gamma = |det P~|^(-1/16), one 16 x 16
//                  factorisation per chunk.
//  * carry scan    its own launch between the passes: a warp per group of G
//                  chunk totals scans the group (inclusive in-group prefixes
//                  and the group total, fp64 on the tensor cores, mma.sync
//                  m8n8k4) and counts the group total in one level up (an
//                  atomic counter); the last warp of a group there scans that
//                  one, up to the top, which is scanned from S0 into
//                  exclusive carries.  No warp waits for another.
//  * apply pass    each chain's first stage brings the chain's carry factors
//                  (the top carry and one in-group prefix per level), their
//                  product is formed in fp64; per stage of 8 tokens the
//                  determinant scales come from 8 LU factorisations at once
//                  (4 lanes per token), then S_t = S_{t-1} + S_{t-1} F_t runs
//                  from the carry and every S_t is written.  Per token·head
//                  the path moves x twice and S once.
//
// Split-tf32 ("3xTF32", after Ootomo and Yokota, 2022): x = hi + lo with hi
// x rounded to tf32 (sign, exponent, 10 mantissa bits) and lo = x - hi exact
// in fp32; a b ~ a_lo b_hi + a_hi b_lo + a_hi b_hi.
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "mru_internal.cuh"

namespace mru {
namespace n16 {
namespace {

constexpr int N = 16;
constexpr int NN = N * N;
constexpr unsigned FULL = 0xffffffffu;

// Pipeline geometry.  Reduce: 4-token stages, three per warp, 8 warps a CTA
// (2 CTAs per SM).  Apply: 8-token stages (one LU round per stage; a stage
// also holds a chain's carry factors, at most 7 KB), two per warp, 4 warps a
// CTA (3 CTAs per SM).
constexpr int RST = 4, RNS = 3, RWARPS = 8;
constexpr int AST = 8, ANS = 2, AWARPS = 4;

template <int ST, int NS>
struct WarpSmem {
    float stage[NS][ST * NN];          // token slices (swizzled) or a chain's carry factors
    float scratch[NN];                 // chunk product (reduce), carry (apply)
    float2 cd[ST];                     // per token: (c alpha, diagonal term of F)
};
using RSmem = WarpSmem<RST, RNS>;      // 13,344 bytes
using ASmem = WarpSmem<AST, ANS>;      // 17,472 bytes

// Word offsets of the carry factors in an apply stage: top carry E (fp64),
// then R_0 (fp32), R_1, R_2 (fp64).
constexpr int CF_E = 0, CF_R0 = 2 * NN, CF_R1 = 3 * NN;
static_assert(CF_R1 + 2 * 2 * NN <= AST * NN, "carry factors must fit one apply stage");

// Word offset of element (row, col) of a token slice in shared memory: row
// pairs form 128-byte lines of eight 16-byte granules, and granule j of line
// l sits at j ^ 2 (l & 3).  The tensor-core fragment reads below are then
// free of bank conflicts without padding the rows.
__device__ __forceinline__ int swz(int row, int col)
{
    const int line = row >> 1;
    const int gran = (((row & 1) << 2) | (col >> 2)) ^ ((line & 3) << 1);
    return (line << 5) | (gran << 2) | (col & 3);
}

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

// hi = v rounded to the nearest tf32 (ties away from zero: the magnitude
// bits plus half a unit of the 10th mantissa bit, then truncated), lo = v - hi.
// A truncated hi would leave every lo with the sign of v and bias the
// dropped lo * lo terms; rounded, they average out.
__device__ __forceinline__ void split_tf32(float v, uint32_t& hi, uint32_t& lo)
{
    const uint32_t h = (__float_as_uint(v) + 0x1000u) & 0xffffe000u;
    hi = h;
    lo = __float_as_uint(v - __uint_as_float(h));
}

// D = A B (+ 0), m16n8k8, tf32 operands, fp32 accumulate.
__device__ __forceinline__ void mma_tf32_first(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(0.0f));
}
// D += A B.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// D += A B, m8n8k4, fp64 throughout.
__device__ __forceinline__ void mma_f64(double (&d)[2], double a, double b)
{
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
                 : "+d"(d[0]), "+d"(d[1])
                 : "d"(a), "d"(b));
}

// ---- per-token determinant scales ------------------------------------------

// Rows r + (16 / R) lr of a 16 x 16 matrix, scale * value (+ I when
// plus_i), from a swizzled token slice (stride 0) or rows `stride` words
// apart.
template <int R>
__device__ __forceinline__ void load_rows(float (&e)[R][N], const float* src, int stride, int r, float scale,
                                          bool plus_i)
{
    constexpr int W = N / R;
#pragma unroll
    for (int lr = 0; lr < R; ++lr) {
        const int i = W * lr + r;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const float4 v = *reinterpret_cast<const float4*>(src + (stride ? i * stride + 4 * c4 : swz(i, 4 * c4)));
            e[lr][4 * c4 + 0] = scale * v.x + ((plus_i && i == 4 * c4 + 0) ? 1.0f : 0.0f);
            e[lr][4 * c4 + 1] = scale * v.y + ((plus_i && i == 4 * c4 + 1) ? 1.0f : 0.0f);
            e[lr][4 * c4 + 2] = scale * v.z + ((plus_i && i == 4 * c4 + 2) ? 1.0f : 0.0f);
            e[lr][4 * c4 + 3] = scale * v.w + ((plus_i && i == 4 * c4 + 3) ? 1.0f : 0.0f);
        }
    }
}

__device__ __forceinline__ float rcp_approx(float v)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(r) : "f"(v));
    return r;
}

// |det(I + e)| of one 16 x 16 matrix held by a group of 16 / R lanes (lane r
// of the group owns rows r + (16 / R) lr, lr < R, in e[lr][0..15]),
// eliminated on e alone without pivoting: prod |1 + delta_k|, an fp32
// product of 16 factors near 1 (relative error about 1e-7: the scale
// c = |det|^(-1/16) it gives is good to about 1e-8).  ok = false when a
// pivot |1 + delta_k| < 0.5.  All lanes of the warp call it (the shuffles
// span the warp).
template <int R>
__device__ __forceinline__ float lu_near_identity(float (&e)[R][N], int r, bool& ok)
{
    constexpr int W = N / R;
    float prod = 1.0f;
    ok = true;
#pragma unroll
    for (int k = 0; k < N; ++k) {
        const int kr = k / W, owner = k % W;
        float prow[N];
#pragma unroll
        for (int j = k; j < N; ++j) prow[j] = __shfl_sync(FULL, e[kr][j], owner, W);
        const float pk = 1.0f + prow[k];
        if (!(fabsf(pk) >= 0.5f)) ok = false;
        prod *= pk;
        const float rk = rcp_approx(pk);
#pragma unroll
        for (int lr = 0; lr < R; ++lr) {
            if (W * lr + W - 1 <= k) continue;    // no row of this slot is below k
            const int i = W * lr + r;
            if (i > k) {
                const float l = e[lr][k] * rk;
#pragma unroll
                for (int j = k + 1; j < N; ++j) e[lr][j] = fmaf(-l, prow[j], e[lr][j]);
            }
        }
    }
    return fabsf(prod);
}

struct LogDet {
    double ld;        // log|det|, summed in fp64
    bool singular;
};

// log|det(W)| with partial pivoting, W = scale * src (+ I when plus_i) loaded
// here (same ownership of rows as lu_near_identity).  The fallback for
// matrices far from the identity: kept out of line, off the hot path's
// instruction footprint.
template <int R>
__device__ __noinline__ LogDet lu_pivoted(const float* src, int stride, int r, float scale, bool plus_i)
{
    constexpr int W = N / R;
    float e[R][N];
    load_rows<R>(e, src, stride, r, scale, plus_i);
    LogDet out;
    out.ld = 0.0;
    out.singular = false;
#pragma unroll
    for (int k = 0; k < N; ++k) {
        const int kr = k / W, owner = k % W;
        float best = -1.0f;
        int bi = k;
#pragma unroll
        for (int lr = 0; lr < R; ++lr) {
            const int i = W * lr + r;
            const float a = fabsf(e[lr][k]);
            if (i >= k && a > best) { best = a; bi = i; }
        }
#pragma unroll
        for (int o = 1; o < W; o <<= 1) {
            const float ob = __shfl_xor_sync(FULL, best, o, W);
            const int oi = __shfl_xor_sync(FULL, bi, o, W);
            if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
        }
        if (!(best > 0.0f)) out.singular = true;
        // swap rows k and bi (row i lives in lane i % W, slot i / W);
        // unconditional (a no-op when bi == k) to keep the warp converged
        const int pr = bi / W, powner = bi % W;
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float vk = 0.0f, vp = 0.0f;
#pragma unroll
            for (int lr = 0; lr < R; ++lr) {
                if (lr == kr) vk = e[lr][j];
                if (lr == pr) vp = e[lr][j];
            }
            const float rowk = __shfl_sync(FULL, vk, owner, W);
            const float rowp = __shfl_sync(FULL, vp, powner, W);
#pragma unroll
            for (int lr = 0; lr < R; ++lr) {
                if (lr == kr && r == owner) e[lr][j] = rowp;
                if (lr == pr && r == powner) e[lr][j] = rowk;
            }
        }
        float prow[N];
#pragma unroll
        for (int j = k; j < N; ++j) prow[j] = __shfl_sync(FULL, e[kr][j], owner, W);
        const float pk = prow[k];
        out.ld += log(fabs((double)pk));
        const float rk = (pk != 0.0f) ? 1.0f / pk : 0.0f;
#pragma unroll
        for (int lr = 0; lr < R; ++lr) {
            if (W * lr + W - 1 <= k) continue;
            const int i = W * lr + r;
            if (i > k) {
                const float l = e[lr][k] * rk;
#pragma unroll
                for (int j = k + 1; j < N; ++j) e[lr][j] = fmaf(-l, prow[j], e[lr][j]);
            }
        }
    }
    return out;
}

// c - 1 = |det W|^(-1/16) - 1 for the matrix at src, W = scale * value
// (+ I where plus_i), by the group of 16 / R lanes.  near (the same for the
// whole warp: it selects code with full-warp shuffles) tries the
// near-identity elimination first (W = I + e; fp32: |det| = 1 + u,
// c - 1 = expm1(-log1p(u) / 16)); the pivoted one runs where any group of the
// warp needs it.  singular: det W = 0 (or not finite).
template <int R>
__device__ __forceinline__ float det_scale_m1(const float* src, int stride, int r, float scale, bool near,
                                              bool plus_i, bool& singular)
{
    bool ok = false;
    float cm1 = 0.0f;
    singular = false;
    if (near) {
        float e[R][N];
        load_rows<R>(e, src, stride, r, scale, false);
        const float ad = lu_near_identity<R>(e, r, ok);
        cm1 = expm1f(-log1pf(ad - 1.0f) * (1.0f / N));
    }
    if (__any_sync(FULL, !ok)) {
        __syncwarp();
        const LogDet q = lu_pivoted<R>(src, stride, r, scale, plus_i);
        if (!ok) {
            singular = q.singular || !isfinite(q.ld);
            cm1 = (float)expm1(-q.ld / N);
        }
    }
    if (!isfinite(cm1) || cm1 <= -1.0f) singular = true;
    return cm1;
}

// The per-token scalars of F = ca M + dv I for the live slots of a stage
// (bit s of live_mask: slot s holds a token), written to cd: one LU
// factorisation per slot, 32 / ST lanes each, in the determinant-corrected
// mode; the constants (alpha, 0 or -1) otherwise.  A singular token sets the
// status bit and keeps X = I.
template <int ST>
__device__ __forceinline__ void stage_scalars(const KParams& p, float2* cd, const float* xs, unsigned live_mask,
                                              int lane, uint32_t* status)
{
    constexpr int R = N * ST / 32, W = N / R;
    const int grp = lane / W, r = lane % W;
    const bool live = (live_mask >> grp) & 1u;
    float ca = p.alpha, dv = p.add_identity ? 0.0f : -1.0f;
    if (p.mode == MRU_MODE_DETNORM) {
        // idle groups factorise I (scale 0, plus I)
        bool singular = false;
        const float cm1 = det_scale_m1<R>(xs + grp * NN, 0, r, live ? p.alpha : 0.0f, p.add_identity != 0,
                                          p.add_identity || !live, singular);
        if (singular) {
            if (live && r == 0) atomicOr(status, STATUS_SINGULAR);
            ca = 0.0f;                       // output unspecified; keep X = I
            dv = 0.0f;
        } else {
            ca = (1.0f + cm1) * p.alpha;
            dv = p.add_identity ? cm1 : -1.0f;
        }
    }
    if (r == 0) cd[grp] = make_float2(ca, dv);
    __syncwarp();
}

// F = X - I = 2 (I - A)^-1 A of the Cayley map X = (I - A)^-1 (I + A),
// A = alpha (M - M^T) / 2, for the live slots of a stage (bit s of live_mask:
// slot s holds a token; slot 0 always does), written over the slots' slices
// (same swizzled layout).  Gauss-Jordan elimination on
// [I - A | 2A] (rows of 32 entries), 8 lanes per token (lane r: rows r and
// r + 8), 4 tokens per round; no pivoting: the symmetric part of I - A is I,
// and every Schur complement keeps a symmetric part of at least I, so each
// pivot is at least 1.  The right half ends as F.
template <int ST>
__device__ __forceinline__ void stage_cayley(float alpha, float* xs, unsigned live_mask, int lane)
{
    static_assert(ST % 4 == 0, "whole rounds of 4 tokens");
    const int grp = lane >> 3, r = lane & 7;
    const float ha = 0.5f * alpha;
#pragma unroll 1
    for (int rd = 0; rd < ST / 4; ++rd) {
        const int tk = 4 * rd + grp;
        const bool live = (live_mask >> tk) & 1u;
        float* ms = xs + (live ? tk : 0) * NN;          // idle groups eliminate slot 0's copy, not stored
        float w[2][2 * N];
#pragma unroll
        for (int lr = 0; lr < 2; ++lr) {
            const int i = r + 8 * lr;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 v = *reinterpret_cast<const float4*>(ms + swz(i, 4 * c4));
                const float mv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * c4 + e;
                    const float a = ha * (mv[e] - ms[swz(j, i)]);
                    w[lr][j] = (i == j ? 1.0f : 0.0f) - a;
                    w[lr][N + j] = 2.0f * a;
                }
            }
        }
        __syncwarp();                                    // every read of M before any write of F
#pragma unroll
        for (int k = 0; k < N; ++k) {
            const int kr = k / 8, owner = k % 8;
            float prow[2 * N];
#pragma unroll
            for (int j = k; j < 2 * N; ++j) prow[j] = __shfl_sync(FULL, w[kr][j], owner, 8);
            const float rk = 1.0f / prow[k];
#pragma unroll
            for (int lr = 0; lr < 2; ++lr) {
                const int i = r + 8 * lr;
                if (i == k) {
#pragma unroll
                    for (int j = k + 1; j < 2 * N; ++j) w[lr][j] = prow[j] * rk;
                } else {
                    const float l = w[lr][k] * rk;
#pragma unroll
                    for (int j = k + 1; j < 2 * N; ++j) w[lr][j] = fmaf(-l, prow[j], w[lr][j]);
                }
            }
        }
        if (live) {
#pragma unroll
            for (int lr = 0; lr < 2; ++lr) {
                const int i = r + 8 * lr;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    *reinterpret_cast<float4*>(ms + swz(i, 4 * c4)) =
                        make_float4(w[lr][N + 4 * c4], w[lr][N + 4 * c4 + 1], w[lr][N + 4 * c4 + 2],
                                    w[lr][N + 4 * c4 + 3]);
            }
        }
        __syncwarp();
    }
}

// ---- the token chain (tf32 split, accumulator-resident state) -------------

// B fragments (split) of F = ca M + dv I for one token, with the contraction
// index permuted (slot q <-> row 8kt + 2q, slot q + 4 <-> row 8kt + 2q + 1),
// and F at this lane's accumulator positions.
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
            const float v0 = fmaf(ca, xs[swz(8 * kt + 2 * q, 8 * nt + g)], kt == nt ? d0 : 0.0f);
            const float v1 = fmaf(ca, xs[swz(8 * kt + 2 * q + 1, 8 * nt + g)], kt == nt ? d1 : 0.0f);
            split_tf32(v0, f.bh[kt][nt][0], f.bl[kt][nt][0]);
            split_tf32(v1, f.bh[kt][nt][1], f.bl[kt][nt][1]);
        }
    if (want_fd) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const float2 xv = *reinterpret_cast<const float2*>(xs + swz(g + 8 * h8, 8 * nt + 2 * q));
                f.fd[nt][2 * h8 + 0] = fmaf(ca, xv.x, h8 == nt ? d0 : 0.0f);
                f.fd[nt][2 * h8 + 1] = fmaf(ca, xv.y, h8 == nt ? d1 : 0.0f);
            }
    }
}

// acc = init + A F with A the 16 x 16 state held in accumulator layout
// (Ad); init is zero (Zero) or F itself at the accumulator positions (the
// reduce pass's F + Q F).  One accumulator per column tile: the six split
// products go in from the smallest (lo hi, hi lo) to the largest (hi hi).
template <bool Zero>
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
        if (Zero) {
            mma_tf32_first(acc[nt], al[0], f.bh[0][nt]);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = f.fd[nt][i];
            mma_tf32(acc[nt], al[0], f.bh[0][nt]);
        }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) mma_tf32(acc[nt], al[1], f.bh[1][nt]);
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma_tf32(acc[nt], ah[kt], f.bl[kt][nt]);
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma_tf32(acc[nt], ah[kt], f.bh[kt][nt]);
}

// ---- the exponential map on the tensor cores -------------------------------

// 1 / k! for k = 0 .. 13.
__constant__ float kInvFact[14] = {1.0f, 1.0f, 0.5f, (float)(1.0 / 6.0), (float)(1.0 / 24.0),
                                   (float)(1.0 / 120.0), (float)(1.0 / 720.0), (float)(1.0 / 5040.0),
                                   (float)(1.0 / 40320.0), (float)(1.0 / 362880.0), (float)(1.0 / 3628800.0),
                                   (float)(1.0 / 39916800.0), (float)(1.0 / 479001600.0),
                                   (float)(1.0 / 6227020800.0)};

// B fragments (split, contraction index permuted as in make_frag_f) of a
// symmetric (sign = 1) or skew-symmetric (sign = -1) 16 x 16 matrix held in
// accumulator layout: the fragment needs element (8 kt + 2 q + e, 8 nt + g),
// which is sign times the lane's own (8 nt + g, 8 kt + 2 q + e).
__device__ __forceinline__ void frag_from_acc(const float (&Ad)[2][4], float sign, FragF& f)
{
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) split_tf32(sign * Ad[kt][2 * nt + e], f.bh[kt][nt][e], f.bl[kt][nt][e]);
}

// A 16 x 16 matrix in accumulator layout written to a swizzled slice.
__device__ __forceinline__ void store_acc_swz(float* ms, const float (&Ad)[2][4], int g, int q)
{
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8)
            *reinterpret_cast<float2*>(ms + swz(g + 8 * h8, 8 * nt + 2 * q)) =
                make_float2(Ad[nt][2 * h8], Ad[nt][2 * h8 + 1]);
}

// F = X - I of the exponential map X = exp(A), A = alpha (M - M^T) / 2, for
// the live slots of a stage (bit s of live_mask: slot s holds a token),
// written over the slots' slices in the same swizzled layout.  The whole warp
// works on one token at a time, its 16 x 16 products on the tensor cores in
// split tf32 (the chain's chain_product).
//
// Scaling and squaring (Moler and Van Loan, 1978), with s and the Taylor
// degree m chosen as the generic kernels choose them: B = A / 2^s with
// ||A||_1 / 2^s <= 1/2, m the least degree (at most 12) whose next term
// ||B||^(m+1) / (m+1)! is below 2^-26 ||B||.  exp(B) - I = sum_k B^k / k!
// (k = 1..m) in Horner form over B^2, pairs of odd and even terms:
// H = c_{2p-1} B + c_{2p} B^2, then H <- c_{2i+1} B + c_{2i+2} B^2 + H B^2
// for i = p-2 .. 0 (p = ceil(m / 2), c_k = 1 / k!, c_k = 0 above m), so
// every product has B^2 as its right operand.  B is skew-symmetric and B^2
// symmetric: each lane's accumulator fragment of B (B^2) gives it its
// B-operand fragments of B (B^2) by transposition, with no data exchange.
// The s squarings (I + F)^2 - I = 2 F + F F take F's B-operand fragments
// through the token's own slice (M is no longer needed there).
template <int ST>
__device__ __forceinline__ void stage_expm(float alpha, float* xs, unsigned live_mask, int lane)
{
    const int g = lane >> 2, q = lane & 3;
    const float ha = 0.5f * alpha;
#pragma unroll 1
    for (int tk = 0; tk < ST; ++tk) {
        if (!((live_mask >> tk) & 1u)) continue;
        float* ms = xs + tk * NN;
        float Bd[2][4];                                  // A at this lane's accumulator positions
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const int r = g + 8 * h8, c = 8 * nt + 2 * q;
                const float2 v = *reinterpret_cast<const float2*>(ms + swz(r, c));
                Bd[nt][2 * h8] = ha * (v.x - ms[swz(c, r)]);
                Bd[nt][2 * h8 + 1] = ha * (v.y - ms[swz(c + 1, r)]);
            }
        __syncwarp();                                    // every read of M before the slice is reused
        // ||A||_1: the lane's share of 4 column sums (rows g and g + 8),
        // summed over g, then the largest column
        float cs[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) cs[2 * nt + e] = fabsf(Bd[nt][e]) + fabsf(Bd[nt][2 + e]);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1)
#pragma unroll
            for (int i = 0; i < 4; ++i) cs[i] += __shfl_xor_sync(FULL, cs[i], o);
        float nrm = fmaxf(fmaxf(cs[0], cs[1]), fmaxf(cs[2], cs[3]));
        nrm = fmaxf(nrm, __shfl_xor_sync(FULL, nrm, 1));
        nrm = fmaxf(nrm, __shfl_xor_sync(FULL, nrm, 2));
        int s2 = 0;
        while (nrm > 0.5f && s2 < 64) { nrm *= 0.5f; ++s2; }     // uniform across the warp
        int m = 1;
        float term = nrm;
        while (m < 12 && term * nrm / (float)(m + 1) > 1.4901161e-8f * nrm) {
            term = term * nrm / (float)(m + 1);
            ++m;
        }
        const float sc = ldexpf(1.0f, -s2);
#pragma unroll
        for (int i = 0; i < 8; ++i) (&Bd[0][0])[i] *= sc;
        FragF f;
        frag_from_acc(Bd, -1.0f, f);
        float P[2][4];                                   // B^2
        chain_product<true>(Bd, f, P);
        frag_from_acc(P, 1.0f, f);
        const int pp = (m + 1) >> 1;
        float H[2][4];
        {
            const float c1 = kInvFact[2 * pp - 1], c2 = 2 * pp <= m ? kInvFact[2 * pp] : 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) (&H[0][0])[i] = fmaf(c1, (&Bd[0][0])[i], c2 * (&P[0][0])[i]);
        }
#pragma unroll 1
        for (int k = pp - 2; k >= 0; --k) {
            float acc[2][4];
            chain_product<true>(H, f, acc);              // H B^2
            const float c1 = kInvFact[2 * k + 1], c2 = kInvFact[2 * k + 2];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                (&H[0][0])[i] = fmaf(c1, (&Bd[0][0])[i], c2 * (&P[0][0])[i]) + (&acc[0][0])[i];
        }
#pragma unroll 1
        for (int r = 0; r < s2; ++r) {
            store_acc_swz(ms, H, g, q);
            __syncwarp();
            FragF fh;
            make_frag_f(ms, 1.0f, 0.0f, 0.0f, g, q, fh, false);
            __syncwarp();                                // every read before the next write
            float acc[2][4];
            chain_product<true>(H, fh, acc);             // F F
#pragma unroll
            for (int i = 0; i < 8; ++i) (&H[0][0])[i] = fmaf(2.0f, (&H[0][0])[i], (&acc[0][0])[i]);
        }
        store_acc_swz(ms, H, g, q);
    }
    __syncwarp();
}

// F = X - I of the orthogonal constructions over the slots' slices: Tr = 1
// the Cayley map, Tr = 2 the exponential map.
template <int Tr, int ST>
__device__ __forceinline__ void stage_transform(float alpha, float* xs, unsigned live_mask, int lane)
{
    if (Tr == 1) stage_cayley<ST>(alpha, xs, live_mask, lane);
    else stage_expm<ST>(alpha, xs, live_mask, lane);
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

// ---- fp64 16 x 16 products on the tensor cores (mma.sync m8n8k4) -----------
//
// A warp holds a 16 x 16 fp64 matrix in accumulator layout: lane (g, t)
// (g = lane / 4, t = lane % 4) keeps M[8 mt + g][8 nb + 2 t + h] in
// m[mt][nb][h] -- the same elements the tf32 accumulator layout gives the
// lane.  As the A operand of the next product the contraction index is
// permuted: k-tile kk = 2 nt + h, slot t <-> column 8 nt + 2 t + h.  The B
// operand then holds, per k-tile kk and column tile nb, B[8 (kk / 2) + 2 t +
// kk % 2][8 nb + g].

template <typename T>
struct M16 {
    T m[2][2][2];
};
template <typename T>
struct F16 {
    T b[4][2];
};
using D16 = M16<double>;
using B16 = F16<double>;

__device__ __forceinline__ void d16_zero(D16& a)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) (&a.m[0][0][0])[i] = 0.0;
}

// acc += A B (B converted to fp64 as it is used).  The k-tiles 0-1 and 2-3
// accumulate separately and are added at the end: two dependent mma steps
// per product instead of four.
template <typename T>
__device__ __forceinline__ void d16_mac(const D16& A, const F16<T>& B, D16& acc)
{
    D16 hi;
    d16_zero(hi);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb)
                mma_f64(kk < 2 ? acc.m[mt][nb] : hi.m[mt][nb], A.m[mt][kk >> 1][kk & 1], (double)B.b[kk][nb]);
#pragma unroll
    for (int i = 0; i < 8; ++i) (&acc.m[0][0][0])[i] += (&hi.m[0][0][0])[i];
}

// One row-major 16 x 16 matrix in shared memory as the B operand, in its own
// precision.
template <typename T>
__device__ __forceinline__ void d16_load(const T* src, F16<T>& b, int lane)
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) b.b[kk][nb] = src[(8 * (kk >> 1) + 2 * t + (kk & 1)) * N + 8 * nb + g];
}

// ---- carry scan (its own launch, between the passes) -----------------------
//
// One warp per group of G chunk totals.  The warp copies the group's items
// into its shared memory (rows padded, one round of copies for up to 16
// fp32 items or 8 fp64 ones), applies the per-chunk determinant correction
// when the reduce pass left it (4-lane LU factorisations, 8 at once), and
// scans them on the fp64 tensor cores.  Then it counts itself in at the
// next level's group; the last warp of a group scans that one, and so on up
// to the top, which is scanned from S0.  No warp waits for another.

constexpr int CWARPS = 4;
constexpr int CROW32 = 20;                  // padded row stride of staged fp32 items (words)
constexpr int CROW64 = 18;                  // padded row stride of staged fp64 items (doubles)
constexpr int CRB32 = 16, CRB64 = 8;        // items per staging round
struct CSmem {
    float buf[CRB32 * N * CROW32];          // 20,480 bytes
    float2 gam[CRB32];                      // per staged item: (gamma, gamma - 1)
};
static_assert(CRB64 * N * CROW64 * sizeof(double) <= sizeof(float) * CRB32 * N * CROW32, "fp64 round fits");

template <typename T> struct Stage;
template <> struct Stage<float> {
    static constexpr int RB = CRB32, ROW = CROW32;
};
template <> struct Stage<double> {
    static constexpr int RB = CRB64, ROW = CROW64;
};

// Copies items [0, cnt) of src (row-major 16 x 16) into buf, rows padded.
template <typename T>
__device__ __forceinline__ void stage_items(T* buf, const T* src, int cnt, int lane)
{
    constexpr int GR = N * (int)sizeof(T) / 16;              // 16-byte granules per row
    constexpr int ROW = Stage<T>::ROW;
    for (int gi = lane; gi < cnt * N * GR; gi += 32) {
        const int item = gi / (N * GR), rem = gi % (N * GR), row = rem / GR, c = rem % GR;
        constexpr int PER = 16 / (int)sizeof(T);
        cp_async16(buf + (item * N + row) * ROW + c * PER, src + (int64_t)item * NN + row * N + c * PER);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
}

// gamma_j = |det(I + Q~_j)|^(-1/16) for the cnt staged fp32 items, 4 lanes
// per item, 8 at once (a singular one gets gamma = 0: the apply pass flags
// its token).
__device__ __forceinline__ void stage_gammas(CSmem& sm, int cnt, int lane)
{
    const int grp = lane >> 2, r = lane & 3;
    for (int b0 = 0; b0 < cnt; b0 += 8) {
        const int item = b0 + grp;
        const bool live = item < cnt;
        bool singular = false;
        const float gm1 = det_scale_m1<4>(sm.buf + (live ? item : 0) * N * CROW32, CROW32, r, live ? 1.0f : 0.0f,
                                          true, true, singular);
        if (live && r == 0) sm.gam[item] = singular ? make_float2(0.0f, -1.0f) : make_float2(1.0f + gm1, gm1);
    }
    __syncwarp();
}

// Staged item j as the B operand (and in accumulator layout), gamma T + (gamma - 1) I.
template <typename T>
__device__ __forceinline__ void load_staged(const T* buf, int j, double gm, double gm1, B16& b, D16& a, int lane)
{
    constexpr int ROW = Stage<T>::ROW;
    const int g = lane >> 2, t = lane & 3;
    const T* it = buf + j * N * ROW;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
            const int row = 8 * (kk >> 1) + 2 * t + (kk & 1), col = 8 * nb + g;
            b.b[kk][nb] = gm * (double)it[row * ROW + col] + (row == col ? gm1 : 0.0);
        }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = 8 * mt + g, col = 8 * nb + 2 * t + h;
                a.m[mt][nb][h] = gm * (double)it[row * ROW + col] + (row == col ? gm1 : 0.0);
            }
}

__device__ __forceinline__ void store_pair(float* p, double a, double b) { *reinterpret_cast<float2*>(p) = make_float2((float)a, (float)b); }
__device__ __forceinline__ void store_pair(double* p, double a, double b) { *reinterpret_cast<double2*>(p) = make_double2(a, b); }

template <typename T>
__device__ __forceinline__ void store_acc(T* dst, const D16& a, int lane)
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) store_pair(dst + (8 * mt + g) * N + 8 * nb + 2 * t, a.m[mt][nb][0], a.m[mt][nb][1]);
}

// Scans the m split-form items at in: Top, the exclusive carries E_0 = S0
// (or I), E_{j+1} = E_j (I + T_j) to E; otherwise the inclusive prefixes
// R_j = R_{j-1} + (T_j + R_{j-1} T_j) to R and the last one to tot.
// correct: the items still need their determinant correction (fp32 only).
template <typename Tin, bool Top, typename Tout>
__device__ __forceinline__ void staged_scan(CSmem& sm, const Tin* in, int m, bool correct, const float* S0,
                                            double* E, Tout* R, double* tot, int lane)
{
    constexpr int RB = Stage<Tin>::RB;
    Tin* buf = reinterpret_cast<Tin*>(sm.buf);
    D16 st, acc, Ta;
    B16 Bf;
    if (Top) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = 8 * mt + g, col = 8 * nb + 2 * t + h;
                    st.m[mt][nb][h] = S0 ? (double)S0[row * N + col] : (row == col ? 1.0 : 0.0);
                }
    } else {
        d16_zero(st);
    }
    for (int j0 = 0; j0 < m; j0 += RB) {
        const int cnt = (m - j0 < RB) ? m - j0 : RB;
        __syncwarp();
        stage_items(buf, in + (int64_t)j0 * NN, cnt, lane);
        if (correct) stage_gammas(sm, cnt, lane);
        // the next item's operands load (and convert) while this step's
        // products run
        B16 Bn;
        D16 Tn;
        auto operands = [&](int j, B16& b, D16& a) {
            double gm = 1.0, gm1 = 0.0;
            if (correct) {
                const float2 gg = sm.gam[j];
                gm = (double)gg.x;
                gm1 = (double)gg.y;
            }
            load_staged(buf, j, gm, gm1, b, a, lane);
        };
        operands(0, Bf, Ta);
        for (int j = 0; j < cnt; ++j) {
            if (j + 1 < cnt) operands(j + 1, Bn, Tn);
            if (Top) {
                store_acc(E + (int64_t)(j0 + j) * NN, st, lane);
                acc = st;                              // E_j + E_j T_j
                d16_mac(st, Bf, acc);
                st = acc;
            } else {
                acc = Ta;                              // T_j + R_{j-1} T_j
                d16_mac(st, Bf, acc);
#pragma unroll
                for (int i = 0; i < 8; ++i) (&st.m[0][0][0])[i] += (&acc.m[0][0][0])[i];
                store_acc(R + (int64_t)(j0 + j) * NN, st, lane);
            }
            Bf = Bn;
            Ta = Tn;
        }
    }
    if (!Top) store_acc(tot, st, lane);
}

// Counts the warp in at a counter whose group has `target` members; true for
// the last one.  The fences order this warp's earlier stores before the count
// and the last one's later loads after it.
__device__ __forceinline__ bool arrive(unsigned* ctr, unsigned target, int lane)
{
    __threadfence();
    __syncwarp();
    unsigned old = 0;
    if (lane == 0) old = atomicAdd(ctr, 1u);
    old = __shfl_sync(FULL, old, 0);
    const bool last = old + 1 == target;
    if (last) __threadfence();
    return last;
}

// One warp per group of level 0 (per sequence when the chunk totals are the
// top level already), then up the levels as the last arriver.
__global__ void __launch_bounds__(CWARPS * 32)
k16_carry(KParams p, const float* __restrict__ totals, CarryPlan cp, char* ws, const float* __restrict__ S0)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    CSmem& sm = reinterpret_cast<CSmem*>(smem_raw)[warp];
    const bool correct = p.mode == MRU_MODE_DETNORM && p.add_identity;
    const int64_t per_seq = cp.levels > 0 ? cp.cnt[1] : 1;
    const int64_t unit = (int64_t)blockIdx.x * CWARPS + warp;
    if (unit >= cp.nseq * per_seq) return;
    const int64_t seq = unit / per_seq;
    const float* s0 = S0 ? S0 + seq * NN : nullptr;
    if (cp.levels == 0) {
        const int64_t m = cp.cnt[0];
        staged_scan<float, true, double>(sm, totals + seq * m * NN, (int)m, correct, s0,
                                         reinterpret_cast<double*>(ws + cp.Etop) + seq * m * NN, nullptr, nullptr,
                                         lane);
        return;
    }
    int64_t gi = unit % per_seq;
    for (int l = 0; l < cp.levels; ++l) {
        if (l > 0) {
            const int64_t item = gi;
            gi = item >> cp.gshift;
            const int64_t m = (cp.cnt[l] - (gi << cp.gshift) < cp.G) ? cp.cnt[l] - (gi << cp.gshift) : cp.G;
            unsigned* ctr = reinterpret_cast<unsigned*>(ws + cp.ctr[l]) + seq * cp.cnt[l + 1] + gi;
            if (!arrive(ctr, (unsigned)m, lane)) return;
        }
        const int64_t first = seq * cp.cnt[l] + (gi << cp.gshift);
        const int64_t m = (cp.cnt[l] - (gi << cp.gshift) < cp.G) ? cp.cnt[l] - (gi << cp.gshift) : cp.G;
        double* tot = reinterpret_cast<double*>(ws + cp.Tot[l]) + (seq * cp.cnt[l + 1] + gi) * NN;
        if (l == 0)
            staged_scan<float, false, float>(sm, totals + first * NN, (int)m, correct, nullptr, nullptr,
                                             reinterpret_cast<float*>(ws + cp.R[0]) + first * NN, tot, lane);
        else
            staged_scan<double, false, double>(sm, reinterpret_cast<const double*>(ws + cp.Tot[l - 1]) + first * NN,
                                               (int)m, false, nullptr, nullptr,
                                               reinterpret_cast<double*>(ws + cp.R[l]) + first * NN, tot, lane);
    }
    const int64_t m = cp.cnt[cp.levels];
    unsigned* ctr = reinterpret_cast<unsigned*>(ws + cp.ctr[cp.levels]) + seq;
    if (!arrive(ctr, (unsigned)m, lane)) return;
    staged_scan<double, true, double>(sm, reinterpret_cast<const double*>(ws + cp.Tot[cp.levels - 1]) + seq * m * NN,
                                      (int)m, false, s0, reinterpret_cast<double*>(ws + cp.Etop) + seq * m * NN,
                                      nullptr, nullptr, lane);
}

// ---- chains and the stage feed ---------------------------------------------

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

// The producer side of a warp's pipeline: the next stage to copy, along the
// warp's chains.  Apply: a chain's first stage is its carry factors.
template <bool Apply, int ST>
struct Feed {
    int64_t chain, stride, nchains, tok;
    int64_t t, tend;
    const float* xb;
    // carry factors (apply): top carry, and per level the in-group prefix
    // before this chain's item (null for the first item of a group)
    const double* E;
    const void* Rf[kCarryLevels];
    bool carry_next;
    // single-chunk problems (one chain per sequence): the carry is S0 (fp32)
    // or I, read directly; no carry scan ran
    bool direct;
    const float* s0;
    const float* s0row;

    __device__ __forceinline__ void set(const KParams& p, const float* x, const CarryPlan& cp, const char* ws)
    {
        if (chain >= nchains) return;
        const Chain c = chain_at(p, chain);
        xb = x + (c.b * p.L * p.H + c.h) * NN;
        t = c.tbeg;
        tend = c.tend;
        if (Apply && direct) {
            s0row = s0 ? s0 + (c.b * p.H + c.h) * NN : nullptr;
            carry_next = true;
        } else if (Apply) {
            const int64_t seq = c.b * p.H + c.h;
            int64_t i = c.k;
#pragma unroll
            for (int l = 0; l < kCarryLevels; ++l) {
                Rf[l] = nullptr;
                if (l < cp.levels) {
                    if (i & (cp.G - 1)) {
                        const size_t esz = l == 0 ? sizeof(float) : sizeof(double);
                        Rf[l] = ws + cp.R[l] + (size_t)((seq * cp.cnt[l] + i - 1) * NN) * esz;
                    }
                    i >>= cp.gshift;
                }
            }
            E = reinterpret_cast<const double*>(ws + cp.Etop) + (seq * cp.cnt[cp.levels] + i) * NN;
            carry_next = true;
        }
    }

    // Copies the next stage into dst (nothing once the chains are done) and
    // commits a cp.async group either way.
    __device__ __forceinline__ void issue(float* dst, int lane, const KParams& p, const float* x,
                                          const CarryPlan& cp, const char* ws)
    {
        if (chain < nchains) {
            if (Apply && carry_next && direct) {
                if (s0row) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) cp_async16(dst + CF_E + 4 * (lane + 32 * i), s0row + 4 * (lane + 32 * i));
                }
                carry_next = false;
            } else if (Apply && carry_next) {
                const char* E8 = reinterpret_cast<const char*>(E);
#pragma unroll
                for (int i = 0; i < 4; ++i) cp_async16(dst + CF_E + 4 * (lane + 32 * i), E8 + 16 * (lane + 32 * i));
                if (Rf[0]) {
                    const char* r8 = reinterpret_cast<const char*>(Rf[0]);
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        cp_async16(dst + CF_R0 + 4 * (lane + 32 * i), r8 + 16 * (lane + 32 * i));
                }
#pragma unroll
                for (int l = 1; l < kCarryLevels; ++l)
                    if (Rf[l]) {
                        const char* r8 = reinterpret_cast<const char*>(Rf[l]);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            cp_async16(dst + CF_R1 + 2 * NN * (l - 1) + 4 * (lane + 32 * i), r8 + 16 * (lane + 32 * i));
                    }
                carry_next = false;
            } else {
                const int nt = (tend - t < ST) ? (int)(tend - t) : ST;
#pragma unroll
                for (int i = 0; i < ST * 2; ++i) {     // 64 granules a slice, 2 per lane
                    const int gi = lane + 32 * i;
                    const int j = gi >> 6, gr = gi & 63, row = gr >> 2, c4 = gr & 3;
                    if (j < nt) cp_async16(dst + j * NN + swz(row, 4 * c4), xb + (t + j) * tok + row * N + 4 * c4);
                }
                t += ST;
                if (t >= tend) {
                    chain += stride;
                    set(p, x, cp, ws);
                }
            }
        }
        cp_async_commit();
    }
};

// The chain's carry C = E (I + R_{levels-1}) ... (I + R_0) in fp64 (factors
// absent for the first item of a group skipped), rounded to fp32 into
// accumulator layout Sd; in = the carry stage.
__device__ __forceinline__ void form_carry(const float* in, const CarryPlan& cp, int64_t k, int lane,
                                           float (&Sd)[2][4])
{
    D16 C, acc;
    {
        const double* sE = reinterpret_cast<const double*>(in + CF_E);
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const double2 v = *reinterpret_cast<const double2*>(sE + (8 * mt + g) * N + 8 * nb + 2 * t);
                C.m[mt][nb][0] = v.x;
                C.m[mt][nb][1] = v.y;
            }
    }
    for (int l = cp.levels - 1; l >= 0; --l) {
        if (((k >> (cp.gshift * l)) & (cp.G - 1)) == 0) continue;
        acc = C;                                   // C (I + R_l)
        if (l == 0) {
            F16<float> Bf;
            d16_load(in + CF_R0, Bf, lane);
            d16_mac(C, Bf, acc);
        } else {
            B16 Bf;
            d16_load(reinterpret_cast<const double*>(in + CF_R1 + 2 * NN * (l - 1)), Bf, lane);
            d16_mac(C, Bf, acc);
        }
        C = acc;
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int h = 0; h < 2; ++h) Sd[nb][2 * mt + h] = (float)C.m[mt][nb][h];
}

// The carry of a single-chunk problem: S0 as staged (fp32, row-major) or I.
__device__ __forceinline__ void direct_carry(const float* in, bool has_s0, int lane, float (&Sd)[2][4])
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = 8 * mt + g, col = 8 * nb + 2 * t + h;
                Sd[nb][2 * mt + h] = has_s0 ? in[CF_E + row * N + col] : (row == col ? 1.0f : 0.0f);
            }
}

// ---- kernels ----------------------------------------------------------------

// Reduce pass: chunk totals (split form).  With PerToken (the corrected mode
// without the identity, whose uncorrected products alpha M could leave the
// fp32 range) the chain takes every token's scale as it goes; otherwise it
// runs on the uncorrected matrices and the carry kernel applies the
// determinant correction of each total.  With an orthogonal construction
// (Tr 1 or 2) and fout non-null, every token's F = X - I is also written to
// fout (x's layout), so that the apply pass reads F instead of forming it
// again.  CTA 0 also zeroes the carry scan's counters (the carry kernel runs
// after this launch).
template <bool PerToken, int Tr = 0>
__global__ void __launch_bounds__(RWARPS * 32, 2)
k16_reduce(KParams p, const float* __restrict__ x, float* __restrict__ totals, unsigned* ctr, int64_t nctr,
           uint32_t* status, float* __restrict__ fout)
{
    if (blockIdx.x == 0)
        for (int64_t i = threadIdx.x; i < nctr; i += blockDim.x) ctr[i] = 0u;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    RSmem& sm = reinterpret_cast<RSmem*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * RWARPS + warp, stride = (int64_t)gridDim.x * RWARPS;
    const int g = lane >> 2, q = lane & 3;
    const float m0 = (g == 2 * q) ? 1.0f : 0.0f;         // diagonal positions of this lane's fragments
    const float m1 = (g == 2 * q + 1) ? 1.0f : 0.0f;
    Feed<false, RST> feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = p.H * NN;
    const CarryPlan nocp = {};            // the reduce feed reads no carry factors
    feed.set(p, x, nocp, nullptr);
#pragma unroll
    for (int s = 0; s < RNS - 1; ++s) feed.issue(sm.stage[s], lane, p, x, nocp, nullptr);
    int cs = 0, ps = RNS - 1;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        float Qd[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) Qd[nt][i] = 0.0f;
        for (int64_t t0 = c.tbeg; t0 < c.tend; t0 += RST) {
            feed.issue(sm.stage[ps], lane, p, x, nocp, nullptr);
            ps = (ps + 1 == RNS) ? 0 : ps + 1;
            cp_async_wait<RNS - 1>();
            __syncwarp();
            const float* xs = sm.stage[cs];
            const int nt = (c.tend - t0 < RST) ? (int)(c.tend - t0) : RST;
            float ca = p.alpha, dv = p.add_identity ? 0.0f : -1.0f;
            if (PerToken) stage_scalars<RST>(p, sm.cd, xs, (1u << nt) - 1u, lane, status);
            if (Tr != 0) {                                 // F itself now sits where M was
                stage_transform<Tr, RST>(p.alpha, sm.stage[cs], (1u << nt) - 1u, lane);
                ca = 1.0f;
                dv = 0.0f;
                if (fout) {                                // F to HBM, x's layout (one copy per slice)
                    float* fb = fout + (c.b * p.L * p.H + c.h) * NN + t0 * feed.tok;
#pragma unroll
                    for (int i = 0; i < RST * 2; ++i) {
                        const int gi = lane + 32 * i;
                        const int j = gi >> 6, gr = gi & 63, row = gr >> 2, c4 = gr & 3;
                        if (j < nt)
                            *reinterpret_cast<float4*>(fb + j * feed.tok + row * N + 4 * c4) =
                                *reinterpret_cast<const float4*>(xs + j * NN + swz(row, 4 * c4));
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < RST; ++j) {
                if (j < nt) {
                    if (PerToken) {
                        const float2 cdj = sm.cd[j];
                        ca = cdj.x;
                        dv = cdj.y;
                    }
                    FragF f;
                    make_frag_f(xs + j * NN, ca, m0 * dv, m1 * dv, g, q, f, true);
                    float acc[2][4];
                    chain_product<false>(Qd, f, acc);         // F + Q F
#pragma unroll
                    for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                        for (int i = 0; i < 4; ++i) Qd[n2][i] += acc[n2][i];
                }
            }
            __syncwarp();
            cs = (cs + 1 == RNS) ? 0 : cs + 1;
        }
        store_d(totals + ((c.b * p.H + c.h) * p.K + c.k) * NN, Qd, g, q);
    }
}

// Apply pass: per chain the carry from the carry scan's factors, then
// S_t = S_{t-1} + S_{t-1} F_t from S = carry, every S_t written, with the
// per-token determinant scales factorised here.  Tr = 3: x holds F = X - I
// already (the reduce pass wrote it), taken with scale 1 and no diagonal
// term.
template <bool Direct, int Tr = 0>
__global__ void __launch_bounds__(AWARPS * 32, 3)
k16_apply(KParams p, const float* __restrict__ x, CarryPlan cp, const char* ws, float* __restrict__ S_out,
          uint32_t* status, const float* __restrict__ S0)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    ASmem& sm = reinterpret_cast<ASmem*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * AWARPS + warp, stride = (int64_t)gridDim.x * AWARPS;
    const int64_t tok = p.H * NN;
    const int g = lane >> 2, q = lane & 3;
    const float m0 = (g == 2 * q) ? 1.0f : 0.0f;
    const float m1 = (g == 2 * q + 1) ? 1.0f : 0.0f;
    Feed<true, AST> feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = tok;
    feed.direct = Direct;
    feed.s0 = S0;
    feed.set(p, x, cp, ws);
#pragma unroll
    for (int s = 0; s < ANS - 1; ++s) feed.issue(sm.stage[s], lane, p, x, cp, ws);
    int cs = 0, ps = ANS - 1;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        float Sd[2][4];
        feed.issue(sm.stage[ps], lane, p, x, cp, ws);
        ps = (ps + 1 == ANS) ? 0 : ps + 1;
        cp_async_wait<ANS - 1>();
        __syncwarp();
        if (Direct) direct_carry(sm.stage[cs], S0 != nullptr, lane, Sd);
        else form_carry(sm.stage[cs], cp, c.k, lane, Sd);
        __syncwarp();
        cs = (cs + 1 == ANS) ? 0 : cs + 1;
        float* ob = S_out + (c.b * p.L * p.H + c.h) * NN;
        for (int64_t t0 = c.tbeg; t0 < c.tend; t0 += AST) {
            feed.issue(sm.stage[ps], lane, p, x, cp, ws);
            ps = (ps + 1 == ANS) ? 0 : ps + 1;
            cp_async_wait<ANS - 1>();
            __syncwarp();
            const float* xs = sm.stage[cs];
            const int nt = (c.tend - t0 < AST) ? (int)(c.tend - t0) : AST;
            if (Tr == 1 || Tr == 2) {                      // F itself now sits where M was
                stage_transform<Tr, AST>(p.alpha, sm.stage[cs], (1u << nt) - 1u, lane);
                if (lane < AST) sm.cd[lane] = make_float2(1.0f, 0.0f);
                __syncwarp();
            } else if (Tr == 3) {
                if (lane < AST) sm.cd[lane] = make_float2(1.0f, 0.0f);
                __syncwarp();
            } else {
                stage_scalars<AST>(p, sm.cd, xs, (1u << nt) - 1u, lane, status);
            }
#pragma unroll
            for (int j = 0; j < AST; ++j) {
                if (j < nt) {
                    const float2 cdj = sm.cd[j];
                    FragF f;
                    make_frag_f(xs + j * NN, cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, f, false);
                    float acc[2][4];
                    chain_product<true>(Sd, f, acc);
#pragma unroll
                    for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                        for (int i = 0; i < 4; ++i) Sd[n2][i] += acc[n2][i];
                    store_d(ob + (t0 + j) * tok, Sd, g, q);
                }
            }
            __syncwarp();
            cs = (cs + 1 == ANS) ? 0 : cs + 1;
        }
    }
}

// ---- single-read fused scan: one persistent launch --------------------------
//
// Warps take items, one chain (b, h, chunk of C tokens) each, from two
// counters that hand them out in chain order (h fastest, then the chunk,
// then b):
//  * reduce item   streams the chunk's slices from HBM (under an L2
//                  evict-last policy, so that the apply item finds them in
//                  L2), factorises every token's determinant in the corrected
//                  mode and records the token's (c alpha, c - 1), runs the
//                  chain on the corrected matrices and writes the chunk total.
//                  The reduce item that completes a group of G chunks of a
//                  sequence scans the group in fp64 (inclusive in-group
//                  prefixes, kept fp32, and the group aggregate), publishes
//                  the aggregate, finds the group's carry by a decoupled
//                  look-back (the aggregates of the earlier groups multiplied
//                  in, from right to left, until an inclusive prefix or S0),
//                  and publishes the carry and the group's inclusive prefix.
//  * apply item    taken only once its group's carry is out: the chain's
//                  carry (group carry times in-group prefix, fp64), then the
//                  chain from it with the recorded scalars, x read a second
//                  time (from L2, evict-first), every S_t written
//                  (evict-first).
// A warp takes the next apply item in chain order when its group's carry is
// out, else the next reduce item.  The only waits -- a look-back on a group
// that no warp has scanned yet, and a warp with nothing to take -- are on
// items of lower chain order, which running warps hold (items are claimed by
// running warps only, reduce tickets in order), so they end; each is bounded
// by a time limit anyway, past which the kernel records STATUS_TIMEOUT,
// raises an abort flag that every warp reads before it takes an item, and
// returns.  Per token-head HBM sees x once and S once.

constexpr int FST = 8, FWARPS = 4;

struct FSmem {
    float stage[2][FST * NN];          // token slices (swizzled), or an apply item's carry factors
    float2 cd[2][FST];                 // per stage: per-token (c alpha, diagonal term of F)
};
// Word offsets of the carry factors in a fused apply stage: the group carry E
// (fp32, full matrix) and the in-group prefix R (fp32, split form).
constexpr int FCF_E = 0, FCF_R = NN;

enum : int { FK_REDUCE = 1, FK_APPLY = 2, FK_DONE = 3 };

struct FCtl {
    unsigned* ctr;        // [0] ticket counter, [1] abort flag
    unsigned* gcnt;       // [seq][NG] reduce items done per group
    unsigned* gflag;      // [seq][NG] 0; 1 aggregate out; 2 carry and inclusive prefix out
    float* tot;           // [seq][K] chunk totals (split form, corrected)
    float* R0;            // [seq][K] inclusive in-group prefixes (split form)
    double* agg;          // [seq][NG] group aggregates (split form)
    double* incl;         // [seq][NG] inclusive prefix through each group (full)
    float* excl;          // [seq][NG] group carries (full)
    float2* cd;           // [seq][Lp] per-token (c alpha, c - 1), corrected mode
    int64_t Lp, NG;
    int64_t lead;         // reduce items handed out before the first apply item
    int32_t gshift;
    uint64_t limit_ns;    // bound on every wait
    int32_t stall_first;  // testing: group 0's carry is never published
};

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void cp_async16_hint(void* smem, const void* gmem, uint64_t pol)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "l"(pol));
}
__device__ __forceinline__ void st_f2_hint(float* p, float a, float b, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(a), "f"(b), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void store_d_hint(float* out, const float (&Ad)[2][4], int g, int q, uint64_t pol)
{
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8)
            st_f2_hint(out + (g + 8 * h8) * N + 8 * nt + 2 * q, Ad[nt][2 * h8], Ad[nt][2 * h8 + 1], pol);
}

// Records a timeout and raises the abort flag.
__device__ __forceinline__ void fused_abort(const FCtl& f, uint32_t* status)
{
    atomicOr(status, STATUS_TIMEOUT);
    atomicExch(f.ctr + 1, 1u);
}

// Ticket -> item.  The schedule: the first `lead` reduce items, then an
// apply item and a reduce item in turn while reduce items remain, then the
// remaining apply items; apply item i thus comes after reduce item
// lead + i - 1.  With lead at least a group of chains (G chunks of every
// head) the apply item's whole group, and every earlier group of its
// sequence, is handed out before it.
__device__ __forceinline__ int fused_decode(unsigned t, int64_t nchains, int64_t lead, int64_t& chain)
{
    const int64_t u = t;
    if (u >= 2 * nchains) return FK_DONE;
    if (u < lead) { chain = u; return FK_REDUCE; }
    const int64_t pairs = nchains - lead;
    if (u < lead + 2 * pairs) {
        const int64_t v = u - lead;
        chain = (v & 1) ? lead + (v >> 1) : (v >> 1);
        return (v & 1) ? FK_REDUCE : FK_APPLY;
    }
    chain = u - nchains;
    return FK_APPLY;
}

__device__ __forceinline__ unsigned* group_flag(const KParams& p, const FCtl& f, const Chain& c)
{
    return f.gflag + (c.b * p.H + c.h) * f.NG + (c.k >> f.gshift);
}

// Waits (lane 0, bounded) until the apply item's group carry is out; false
// on timeout or when the launch is aborting.  `seen` is a flag value read
// earlier (0 when none was).
__device__ bool wait_ready(const unsigned* flag, unsigned seen, const FCtl& f, uint32_t* status)
{
    if (seen == 2u) return true;
    const uint64_t t0 = global_ns();
    unsigned ns = 64;
    for (;;) {
        if (ld_acquire(flag) == 2u) return true;
        if (ld_acquire(f.ctr + 1)) return false;
        if (global_ns() - t0 > f.limit_ns) {
            fused_abort(f, status);
            return false;
        }
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
    }
}

// A 16 x 16 matrix from global memory (bypassing L1) in accumulator layout
// (fp64), full form (plus_i adds I to a split-form matrix).
template <typename T>
__device__ __forceinline__ void d16_ld_acc(const T* src, D16& a, int lane, bool plus_i)
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = 8 * mt + g, col = 8 * nb + 2 * t + h;
                a.m[mt][nb][h] = (double)__ldcg(src + row * N + col) + ((plus_i && row == col) ? 1.0 : 0.0);
            }
}
// The same as the B operand.
template <typename T>
__device__ __forceinline__ void d16_ld_b(const T* src, B16& b, int lane)
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) b.b[kk][nb] = (double)__ldcg(src + (8 * (kk >> 1) + 2 * t + (kk & 1)) * N + 8 * nb + g);
}

// The group scan: R_j = R_{j-1} + (T_j + R_{j-1} T_j) over the m chunk totals
// at tot (fp64; R_j kept fp32 at R), the last one, the aggregate, to agg.
// Operands come straight from L2, two items ahead of the products.
__device__ __noinline__ void fused_group_scan(const float* tot, float* R, double* agg, int m, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    float rb[2][8], ra[2][8];
    auto fetch = [&](int j, float (&b)[8], float (&a)[8]) {
        const float* it = tot + (int64_t)j * NN;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) b[2 * kk + nb] = __ldcg(it + (8 * (kk >> 1) + 2 * t + (kk & 1)) * N + 8 * nb + g);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const float2 v = __ldcg(reinterpret_cast<const float2*>(it + (8 * mt + g) * N + 8 * nb + 2 * t));
                a[4 * mt + 2 * nb] = v.x;
                a[4 * mt + 2 * nb + 1] = v.y;
            }
    };
    fetch(0, rb[0], ra[0]);
    if (m > 1) fetch(1, rb[1], ra[1]);
    D16 st, acc;
    d16_zero(st);
    for (int j = 0; j < m; ++j) {
        B16 Bf;
        const int s = j & 1;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) Bf.b[kk][nb] = (double)rb[s][2 * kk + nb];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                for (int h = 0; h < 2; ++h) acc.m[mt][nb][h] = (double)ra[s][4 * mt + 2 * nb + h];
        if (j + 2 < m) fetch(j + 2, rb[s], ra[s]);
        d16_mac(st, Bf, acc);                          // T_j + R_{j-1} T_j
#pragma unroll
        for (int i = 0; i < 8; ++i) (&st.m[0][0][0])[i] += (&acc.m[0][0][0])[i];
        store_acc(R + (int64_t)j * NN, st, lane);
    }
    store_acc(agg, st, lane);
}

// The decoupled look-back of group gi of one sequence: the carry
// E = E_0 (I + A_0) ... (I + A_{gi-1}), E_0 = S0 (or I), taken from the
// first group j < gi (right to left) whose inclusive prefix is out, the
// aggregates A of the groups in between multiplied in; then the group's
// carry (fp32) and inclusive prefix E (I + A_gi) (fp64) are written and
// published.  pf: 2 KB of this warp's shared memory.  False when a wait ran
// out (or the launch is aborting).
__device__ __noinline__ bool fused_lookback(const FCtl f, int64_t seq, int64_t gi, const float* s0, double* pf,
                                            uint32_t* status, int lane)
{
    const int64_t base = seq * f.NG;
    // P = (I + A_{j+1}) ... (I + A_{gi-1}), full form, in registers and in pf
    D16 P, acc, E;
    {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                for (int h = 0; h < 2; ++h) P.m[mt][nb][h] = (8 * mt + g == 8 * nb + 2 * t + h) ? 1.0 : 0.0;
    }
    store_acc(pf, P, lane);
    __syncwarp();
    bool found = false;
    for (int64_t j = gi - 1; j >= 0; --j) {
        unsigned fl = 0;
        if (lane == 0) {
            const uint64_t t0 = global_ns();
            unsigned ns = 32;
            for (;;) {
                fl = ld_acquire(f.gflag + base + j);
                if (fl >= 1u || ld_acquire(f.ctr + 1)) break;
                if (global_ns() - t0 > f.limit_ns) {
                    fused_abort(f, status);
                    break;
                }
                __nanosleep(ns);
                if (ns < 1024) ns <<= 1;
            }
        }
        fl = __shfl_sync(FULL, fl, 0);
        if (fl == 0u) return false;
        B16 Pb;
        d16_load(pf, Pb, lane);
        if (fl == 2u) {                                    // E = incl_j P
            D16 Ij;
            d16_ld_acc(f.incl + (base + j) * NN, Ij, lane, false);
            d16_zero(E);
            d16_mac(Ij, Pb, E);
            found = true;
            break;
        }
        D16 Aj;                                            // P <- (I + A_j) P = P + A_j P
        d16_ld_acc(f.agg + (base + j) * NN, Aj, lane, false);
        acc = P;
        d16_mac(Aj, Pb, acc);
        P = acc;
        __syncwarp();
        store_acc(pf, P, lane);
        __syncwarp();
    }
    if (!found) {                                          // E = E_0 P
        if (s0) {
            D16 Z;
            B16 Pb;
            d16_load(pf, Pb, lane);
            d16_ld_acc(s0, Z, lane, false);
            d16_zero(E);
            d16_mac(Z, Pb, E);
        } else {
            E = P;
        }
    }
    // the group's carry (fp32) and its inclusive prefix E + E A_gi (fp64)
    store_acc(f.excl + (base + gi) * NN, E, lane);
    B16 Ab;
    d16_ld_b(f.agg + (base + gi) * NN, Ab, lane);
    acc = E;
    d16_mac(E, Ab, acc);
    store_acc(f.incl + (base + gi) * NN, acc, lane);
    __threadfence();
    __syncwarp();
    if (lane == 0 && !(f.stall_first && gi == 0)) st_release(f.gflag + base + gi, 2u);
    return true;
}

// The carry of an apply item, C = E (I + R) in fp64 (R absent for the first
// chunk of a group), rounded to fp32 into accumulator layout.
__device__ __forceinline__ void fused_carry(const float* in, bool has_r, int lane, float (&Sd)[2][4])
{
    D16 C;
    {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const float2 v = *reinterpret_cast<const float2*>(in + FCF_E + (8 * mt + g) * N + 8 * nb + 2 * t);
                C.m[mt][nb][0] = v.x;
                C.m[mt][nb][1] = v.y;
            }
    }
    if (has_r) {
        D16 acc = C;
        F16<float> Rb;
        d16_load(in + FCF_R, Rb, lane);
        d16_mac(C, Rb, acc);
        C = acc;
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int h = 0; h < 2; ++h) Sd[nb][2 * mt + h] = (float)C.m[mt][nb][h];
}

// Stage `s` of item (kind, chain) into buf / cdbuf: for an apply item stage 0
// is the carry factors, then the token stages of FST tokens.
__device__ __forceinline__ void fused_issue(const KParams& p, const FCtl& f, const float* x, int kind,
                                            const Chain& c, int s, float* buf, float2* cdbuf, int lane,
                                            uint64_t pol_x)
{
    const int64_t seq = c.b * p.H + c.h;
    if (kind == FK_APPLY && s == 0) {
        const int64_t gi = c.k >> f.gshift;
        const float* E = f.excl + (seq * f.NG + gi) * NN;
#pragma unroll
        for (int i = 0; i < 2; ++i) cp_async16(buf + FCF_E + 4 * (lane + 32 * i), E + 4 * (lane + 32 * i));
        if (c.k & ((1 << f.gshift) - 1)) {
            const float* R = f.R0 + (seq * p.K + c.k - 1) * NN;
#pragma unroll
            for (int i = 0; i < 2; ++i) cp_async16(buf + FCF_R + 4 * (lane + 32 * i), R + 4 * (lane + 32 * i));
        }
        return;
    }
    const int64_t t0 = c.tbeg + (int64_t)(s - (kind == FK_APPLY ? 1 : 0)) * FST;
    const int nt = (c.tend - t0 < FST) ? (int)(c.tend - t0) : FST;
    const float* xb = x + ((c.b * p.L + t0) * p.H + c.h) * NN;
    const int64_t tok = p.H * NN;
#pragma unroll
    for (int i = 0; i < FST * 2; ++i) {                    // 64 granules a slice, 2 per lane
        const int gi = lane + 32 * i;
        const int j = gi >> 6, gr = gi & 63, row = gr >> 2, c4 = gr & 3;
        if (j < nt) cp_async16_hint(buf + j * NN + swz(row, 4 * c4), xb + j * tok + row * N + 4 * c4, pol_x);
    }
    if (kind == FK_APPLY && p.mode == MRU_MODE_DETNORM && lane < FST / 2)
        cp_async16(cdbuf + 2 * lane, f.cd + seq * f.Lp + t0 + 2 * lane);
}

template <int Tr>
__global__ void __launch_bounds__(FWARPS * 32, 3)
k16_fused(KParams p, FCtl f, const float* __restrict__ x, const float* __restrict__ S0, float* __restrict__ S_out,
          uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    FSmem& sm = reinterpret_cast<FSmem*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int g = lane >> 2, q = lane & 3;
    const float m0 = (g == 2 * q) ? 1.0f : 0.0f;
    const float m1 = (g == 2 * q + 1) ? 1.0f : 0.0f;
    const int G = 1 << f.gshift;
    const bool detnorm = p.mode == MRU_MODE_DETNORM && Tr == 0;
    const uint64_t pol_keep = policy_evict_last(), pol_drop = policy_evict_first();
    const int64_t tok = p.H * NN;

    // the first item
    unsigned tk = 0;
    if (lane == 0) tk = atomicAdd(f.ctr, 1u);
    tk = __shfl_sync(FULL, tk, 0);
    int64_t chain = 0;
    int kind = fused_decode(tk, nchains, f.lead, chain);
    if (kind == FK_DONE) return;
    Chain c = chain_at(p, chain);
    if (kind == FK_APPLY) {
        bool ok = true;
        if (lane == 0) ok = wait_ready(group_flag(p, f, c), 0u, f, status);
        if (!__shfl_sync(FULL, (int)ok, 0)) return;
        __syncwarp();
    }
    unsigned slot = 0;                                     // stream position: stage buffers alternate
    fused_issue(p, f, x, kind, c, 0, sm.stage[0], sm.cd[0], lane, kind == FK_APPLY ? pol_drop : pol_keep);
    cp_async_commit();
    for (;;) {
        // claim the next item now; its ticket is read one stage later and
        // (for an apply item) its group flag at the last stage
        unsigned tk_next = 0, fl_next = 0;
        if (lane == 0) tk_next = atomicAdd(f.ctr, 1u);
        int nkind = FK_DONE;
        int64_t nchain = 0;
        Chain nc = c;
        bool decoded = false, deferred = false;
        const int ntok = (int)(c.tend - c.tbeg);
        const int nst = (ntok + FST - 1) / FST + (kind == FK_APPLY ? 1 : 0);
        const int64_t seq = c.b * p.H + c.h;
        float St[2][4];                                    // the chain's state: Q (reduce) or S (apply)
#pragma unroll
        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
            for (int i = 0; i < 4; ++i) St[n2][i] = 0.0f;
        for (int s = 0; s < nst; ++s) {
            const unsigned cur = slot & 1u, nxt = cur ^ 1u;
            if (s + 1 < nst) {
                fused_issue(p, f, x, kind, c, s + 1, sm.stage[nxt], sm.cd[nxt], lane,
                            kind == FK_APPLY ? pol_drop : pol_keep);
            } else {
                if (!decoded) {
                    nkind = fused_decode(__shfl_sync(FULL, tk_next, 0), nchains, f.lead, nchain);
                    if (nkind != FK_DONE) nc = chain_at(p, nchain);
                }
                // an apply item's carry factors are fetched now only if its
                // group carry is out already; otherwise after this item is
                // finished (waiting here could wait on this very item)
                if (nkind == FK_APPLY) {
                    int ready = 0;
                    if (lane == 0) ready = fl_next == 2u || ld_acquire(group_flag(p, f, nc)) == 2u;
                    deferred = !__shfl_sync(FULL, ready, 0);
                    __syncwarp();
                }
                if (nkind != FK_DONE && !deferred)
                    fused_issue(p, f, x, nkind, nc, 0, sm.stage[nxt], sm.cd[nxt], lane,
                                nkind == FK_APPLY ? pol_drop : pol_keep);
            }
            cp_async_commit();
            cp_async_wait<1>();
            __syncwarp();
            ++slot;
            float* xs = sm.stage[cur];
            if (kind == FK_APPLY && s == 0) {
                fused_carry(xs, (c.k & (G - 1)) != 0, lane, St);
            } else {
                const int64_t t0 = c.tbeg + (int64_t)(s - (kind == FK_APPLY ? 1 : 0)) * FST;
                const int nt = (c.tend - t0 < FST) ? (int)(c.tend - t0) : FST;
                float2* cdv = sm.cd[cur];
                if (Tr != 0) {
                    stage_transform<Tr, FST>(p.alpha, xs, (1u << nt) - 1u, lane);
                    if (lane < FST) cdv[lane] = make_float2(1.0f, 0.0f);
                    __syncwarp();
                } else if (kind == FK_REDUCE) {
                    stage_scalars<FST>(p, cdv, xs, (1u << nt) - 1u, lane, status);
                    if (detnorm && lane < nt) f.cd[seq * f.Lp + t0 + lane] = cdv[lane];
                } else if (!detnorm) {
                    if (lane < FST) cdv[lane] = make_float2(p.alpha, p.add_identity ? 0.0f : -1.0f);
                    __syncwarp();
                }
                // One copy of each chain loop, not unrolled over the stage's
                // tokens (the kernel's code must stay small enough for the
                // instruction cache); the next token's fragments are formed
                // while this token's products run.
                if (kind == FK_REDUCE) {
                    FragF fr;
                    float2 cdj = cdv[0];
                    make_frag_f(xs, cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, fr, true);
#pragma unroll 1
                    for (int j = 0; j < nt; ++j) {
                        float acc[2][4];
                        chain_product<false>(St, fr, acc);        // F + Q F
                        if (j + 1 < nt) {
                            cdj = cdv[j + 1];
                            make_frag_f(xs + (j + 1) * NN, cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, fr, true);
                        }
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) St[n2][i] += acc[n2][i];
                    }
                } else {
                    float* ob = S_out + ((c.b * p.L + t0) * p.H + c.h) * NN;
                    FragF fr;
                    float2 cdj = cdv[0];
                    make_frag_f(xs, cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, fr, false);
#pragma unroll 1
                    for (int j = 0; j < nt; ++j) {
                        float acc[2][4];
                        chain_product<true>(St, fr, acc);         // S F
                        if (j + 1 < nt) {
                            cdj = cdv[j + 1];
                            make_frag_f(xs + (j + 1) * NN, cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, fr, false);
                        }
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) St[n2][i] += acc[n2][i];
                        store_d_hint(ob + j * tok, St, g, q, pol_drop);
                    }
                }
            }
            __syncwarp();
            if (s == 0 && nst > 1) {
                // the next ticket has had this stage to arrive: decode it, and
                // start reading an apply item's group flag
                nkind = fused_decode(__shfl_sync(FULL, tk_next, 0), nchains, f.lead, nchain);
                decoded = true;
                if (nkind != FK_DONE) {
                    nc = chain_at(p, nchain);
                    if (nkind == FK_APPLY && lane == 0) fl_next = ld_acquire(group_flag(p, f, nc));
                }
            }
            if (s + 1 == nst && kind == FK_REDUCE) {
                // the chunk total, then the group's count; the last one scans
                store_d(f.tot + (seq * p.K + c.k) * NN, St, g, q);
                const int64_t gi = c.k >> f.gshift;
                const int64_t first = gi << f.gshift;
                const int m = (p.K - first < G) ? (int)(p.K - first) : G;
                if (arrive(f.gcnt + seq * f.NG + gi, (unsigned)m, lane)) {
                    fused_group_scan(f.tot + (seq * p.K + first) * NN, f.R0 + (seq * p.K + first) * NN,
                                     f.agg + (seq * f.NG + gi) * NN, m, lane);
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) st_release(f.gflag + seq * f.NG + gi, 1u);
                    fused_lookback(f, seq, gi, S0 ? S0 + seq * NN : nullptr, reinterpret_cast<double*>(xs),
                                   status, lane);
                }
            }
        }
        if (nkind == FK_DONE) break;
        if (deferred) {                                    // this item is done: wait for the carry
            bool ok = true;
            if (lane == 0) ok = wait_ready(group_flag(p, f, nc), 0u, f, status);
            if (!__shfl_sync(FULL, (int)ok, 0)) break;
            __syncwarp();
            fused_issue(p, f, x, nkind, nc, 0, sm.stage[slot & 1u], sm.cd[slot & 1u], lane, pol_drop);
            cp_async_commit();
        }
        kind = nkind;
        c = nc;
    }
    cp_async_wait<0>();
}

// ---- backward (vector-Jacobian product) on the tensor cores ----------------
//
// G_t = dL/dS_t (later states included): G_{t-1} = dS_{t-1} + G_t X_t^T and
// dL/dX_t = S_{t-1}^T G_t, the chain rule of S_t = S_{t-1} X_t.  Chunked as
// the generic backward is: a local pass per chunk [t0, t1) (the gradient at
// t0 with nothing entering from the right, and W - I with
// W = X_{t0+1} ... X_{t1}), the generic fp64 right-to-left scan of the chunk
// gradients, and an apply pass per chunk (G from the gradient entering from
// the right down to t0, dX_t, and the construction's chain rule).
// Persistent warps, one chunk at a time, the chunk's tokens in reverse order
// through a cp.async pipeline of 2-token stages (x_t, S_{t-1}, dS_{t-1}); per
// stage the two tokens' determinant scales (16 lanes per LU).  Split-tf32
// products with the matrices in the accumulators:
//   G <- dS_{t-1} + G + G F_t^T        B = F_t^T, read transposed from x_t
//   W^T <- W^T + F_t^T + W^T F_t^T     (local pass; W^T keeps the left
//                                       multiplications of W on the right)
//   dX = S_{t-1}^T G                   G staged through shared memory
// Determinant-corrected chain rule: dXr = c (dX - <dX, Xr> Xr^-T / 16),
// dM = alpha dXr, with Xr^-T = (I + E^T)^-1 (E = alpha M) by Newton-Schulz in
// split form: Y = I + Z, R = I - Y (I + E^T) = -(Z + E^T + Z E^T),
// Z <- Z + R + R Z, from Z = -E^T.  The residual squares every step, from
// at most |E|_F^2, so the least k with (|E|_F^2)^(2^k) <= 2^-20 steps are
// run; all but the last in single tf32 (the iteration corrects what they
// round), the last with Z E^T in split tf32.  |E|_F^2 > 0.8 (far from the
// identity): Gauss-Jordan elimination with partial pivoting on the lanes.

constexpr int BST = 2, BNS = 2, BWARPS = 4;

template <bool Apply>
struct BSmem {
    float x[BNS][BST * NN];                           // slices x_t (swizzled)
    float ds[BNS][BST * NN];                          // dS_{t-1}
    float s[Apply ? BNS : 1][Apply ? BST * NN : 4];   // S_{t-1} (apply pass)
    float stg[NN];                                    // a staged accumulator matrix (swizzled)
    float2 cd[BST];                                   // per token: (c alpha, diagonal term of F)
};

// tf32 of v, rounded to nearest (the high part of split_tf32).
__device__ __forceinline__ uint32_t tf32_rn(float v) { return (__float_as_uint(v) + 0x1000u) & 0xffffe000u; }

// B fragments (split) of F^T for F = ca M + dv I, with the contraction index
// permuted as in make_frag_f, and F^T at this lane's accumulator positions.
__device__ __forceinline__ void make_frag_ft(const float* xs, float ca, float d0, float d1, int g, int q, FragF& f,
                                             bool want_fd)
{
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float v0 = fmaf(ca, xs[swz(8 * nt + g, 8 * kt + 2 * q)], kt == nt ? d0 : 0.0f);
            const float v1 = fmaf(ca, xs[swz(8 * nt + g, 8 * kt + 2 * q + 1)], kt == nt ? d1 : 0.0f);
            split_tf32(v0, f.bh[kt][nt][0], f.bl[kt][nt][0]);
            split_tf32(v1, f.bh[kt][nt][1], f.bl[kt][nt][1]);
        }
    if (want_fd) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                f.fd[nt][2 * h8 + 0] = fmaf(ca, xs[swz(8 * nt + 2 * q, g + 8 * h8)], h8 == nt ? d0 : 0.0f);
                f.fd[nt][2 * h8 + 1] = fmaf(ca, xs[swz(8 * nt + 2 * q + 1, g + 8 * h8)], h8 == nt ? d1 : 0.0f);
            }
    }
}

// acc = A B in single tf32: A the accumulator-resident matrix (permuted
// contraction), b its partner's fragments.
__device__ __forceinline__ void product_tf32(const float (&Ad)[2][4], const uint32_t (&b)[2][2][2], float (&acc)[2][4])
{
    uint32_t a[2][4];
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
        a[kt][0] = tf32_rn(Ad[kt][0]);
        a[kt][1] = tf32_rn(Ad[kt][2]);
        a[kt][2] = tf32_rn(Ad[kt][1]);
        a[kt][3] = tf32_rn(Ad[kt][3]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        mma_tf32_first(acc[nt], a[0], b[0][nt]);
        mma_tf32(acc[nt], a[1], b[1][nt]);
    }
}

// An accumulator matrix into a swizzled shared tile, and back.
__device__ __forceinline__ void stage_acc(float* t, const float (&Ad)[2][4], int g, int q)
{
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8)
            *reinterpret_cast<float2*>(t + swz(g + 8 * h8, 8 * nt + 2 * q)) = make_float2(Ad[nt][2 * h8], Ad[nt][2 * h8 + 1]);
}
__device__ __forceinline__ void unstage_acc(const float* t, float (&Ad)[2][4], int g, int q)
{
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const float2 v = *reinterpret_cast<const float2*>(t + swz(g + 8 * h8, 8 * nt + 2 * q));
            Ad[nt][2 * h8] = v.x;
            Ad[nt][2 * h8 + 1] = v.y;
        }
}
// A 16 x 16 row-major matrix in global memory into / out of accumulator layout.
__device__ __forceinline__ void load_acc(float (&Ad)[2][4], const float* src, int g, int q)
{
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const float2 v = *reinterpret_cast<const float2*>(src + (g + 8 * h8) * N + 8 * nt + 2 * q);
            Ad[nt][2 * h8] = v.x;
            Ad[nt][2 * h8 + 1] = v.y;
        }
}

// dX = S^T G: A = S^T read from the swizzled tile ss (contraction in natural
// order), B = G from the staging tile gs; split tf32, fp32 accumulation.
__device__ __forceinline__ void st_times_g(const float* ss, const float* gs, int g, int q, float (&acc)[2][4])
{
    uint32_t ah[2][4], al[2][4], bh[2][2][2], bl[2][2][2];
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
        split_tf32(ss[swz(8 * kt + q, g)], ah[kt][0], al[kt][0]);
        split_tf32(ss[swz(8 * kt + q, g + 8)], ah[kt][1], al[kt][1]);
        split_tf32(ss[swz(8 * kt + q + 4, g)], ah[kt][2], al[kt][2]);
        split_tf32(ss[swz(8 * kt + q + 4, g + 8)], ah[kt][3], al[kt][3]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            split_tf32(gs[swz(8 * kt + q, 8 * nt + g)], bh[kt][nt][0], bl[kt][nt][0]);
            split_tf32(gs[swz(8 * kt + q + 4, 8 * nt + g)], bh[kt][nt][1], bl[kt][nt][1]);
        }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        mma_tf32_first(acc[nt], al[0], bh[0][nt]);
        mma_tf32(acc[nt], al[1], bh[1][nt]);
    }
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma_tf32(acc[nt], ah[kt], bl[kt][nt]);
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma_tf32(acc[nt], ah[kt], bh[kt][nt]);
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);   // every lane ends with the same sum
    return v;
}

// Z = Xr^-T - I for Xr = I + alpha M (the slice xs) by Gauss-Jordan
// elimination with partial pivoting on [Xr^T | I]: lane i (and i + 16) holds
// row i; Z goes to the accumulator positions through stg.  For tokens far
// from the identity; kept out of line.
__device__ __noinline__ void inverse_t_pivoted(const float* xs, float alpha, float* stg, int lane, float (&Z)[2][4])
{
    const int r = lane & 15, g = lane >> 2, q = lane & 3;
    float a[N], b[N];
#pragma unroll
    for (int j = 0; j < N; ++j) {
        a[j] = fmaf(alpha, xs[swz(j, r)], j == r ? 1.0f : 0.0f);    // Xr^T[r][j] = Xr[j][r]
        b[j] = j == r ? 1.0f : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < N; ++k) {
        float best = r >= k ? fabsf(a[k]) : -1.0f;
        int bi = r;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(FULL, best, o, 16);
            const int oi = __shfl_xor_sync(FULL, bi, o, 16);
            if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
        }
#pragma unroll
        for (int j = 0; j < N; ++j) {                                 // swap rows k and bi
            const float ak = __shfl_sync(FULL, a[j], k, 16), ap = __shfl_sync(FULL, a[j], bi, 16);
            const float bk = __shfl_sync(FULL, b[j], k, 16), bp = __shfl_sync(FULL, b[j], bi, 16);
            if (r == k) { a[j] = ap; b[j] = bp; } else if (r == bi) { a[j] = ak; b[j] = bk; }
        }
        const float pk = __shfl_sync(FULL, a[k], k, 16);
        const float rp = pk != 0.0f ? 1.0f / pk : 0.0f;
        const float f = a[k];
#pragma unroll
        for (int j = 0; j < N; ++j) {
            const float ak = __shfl_sync(FULL, a[j], k, 16) * rp, bk = __shfl_sync(FULL, b[j], k, 16) * rp;
            if (r == k) { a[j] = ak; b[j] = bk; } else { a[j] = fmaf(-f, ak, a[j]); b[j] = fmaf(-f, bk, b[j]); }
        }
    }
    __syncwarp();
    if (lane < 16)
#pragma unroll
        for (int j = 0; j < N; ++j) stg[swz(r, j)] = b[j] - (j == r ? 1.0f : 0.0f);
    __syncwarp();
    unstage_acc(stg, Z, g, q);
    __syncwarp();
}

// Z = (I + E^T)^-1 - I at the accumulator positions, fe = E^T's fragments and
// values, fro2 = |E|_F^2 (the same on every lane); Newton-Schulz as above.
__device__ __forceinline__ void inverse_t_ns(const FragF& fe, float fro2, float* stg, int g, int q, float (&Z)[2][4])
{
    const float l = -log2f(fmaxf(fro2, 1e-30f));
    int k = 1;
    while (k < 6 && (float)(1 << k) * l < 20.0f) ++k;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) Z[nt][i] = -fe.fd[nt][i];
    for (int it = 1; it <= k; ++it) {
        float P[2][4], R[2][4], Qz[2][4];
        if (it == k) chain_product<true>(Z, fe, P);
        else product_tf32(Z, fe.bh, P);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) R[nt][i] = -((Z[nt][i] + fe.fd[nt][i]) + P[nt][i]);
        stage_acc(stg, Z, g, q);
        __syncwarp();
        uint32_t zb[2][2][2];
#pragma unroll
        for (int kt = 0; kt < 2; ++kt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                zb[kt][nt][0] = tf32_rn(stg[swz(8 * kt + 2 * q, 8 * nt + g)]);
                zb[kt][nt][1] = tf32_rn(stg[swz(8 * kt + 2 * q + 1, 8 * nt + g)]);
            }
        __syncwarp();
        product_tf32(R, zb, Qz);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) Z[nt][i] += R[nt][i] + Qz[nt][i];
    }
}

// The producer side of a backward warp's pipeline: the next stage of items
// along the warp's chains.  Items of a chunk [t0, t1): the token after it
// when there is one (only its matrix is used), then t1 - 1 down to t0 (apply)
// or t0 + 1 (local).
template <bool Apply>
struct BFeed {
    int64_t chain, stride, nchains, tok;
    int64_t t, lo, base;

    __device__ __forceinline__ void set(const KParams& p)
    {
        while (chain < nchains) {
            const Chain c = chain_at(p, chain);
            const int64_t hi = c.tend < p.L ? c.tend : c.tend - 1;
            const int64_t l = Apply ? c.tbeg : c.tbeg + 1;
            if (hi >= l) {
                t = hi;
                lo = l;
                base = (c.b * p.L * p.H + c.h) * NN;
                return;
            }
            chain += stride;                 // no items (a one-token chunk at the end, local pass)
        }
    }

    __device__ __forceinline__ void issue(BSmem<Apply>& sm, int slot, int lane, const KParams& p, const float* x,
                                          const float* S, const float* dS)
    {
        if (chain < nchains) {
            const int nt = (t - lo + 1 < BST) ? (int)(t - lo + 1) : BST;
#pragma unroll
            for (int i = 0; i < BST * 2; ++i) {       // 64 granules a tile, 2 per lane
                const int gi = lane + 32 * i;
                const int j = gi >> 6, gr = gi & 63, row = gr >> 2, c4 = gr & 3;
                if (j < nt) {
                    const int64_t tau = t - j;
                    const int so = j * NN + swz(row, 4 * c4);
                    const int64_t go = base + row * N + 4 * c4;
                    cp_async16(&sm.x[slot][so], x + go + tau * tok);
                    if (tau >= 1) {
                        cp_async16(&sm.ds[slot][so], dS + go + (tau - 1) * tok);
                        if (Apply) cp_async16(&sm.s[slot][so], S + go + (tau - 1) * tok);
                    }
                }
            }
            t -= BST;
            if (t < lo) {
                chain += stride;
                set(p);
            }
        }
        cp_async_commit();
    }
};

// dS_{t-1} (a staged tile) added to the accumulator matrix: G = ds + (G + a).
__device__ __forceinline__ void add_ds(const float* dst, const float (&a)[2][4], float (&G)[2][4], int g, int q)
{
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const float2 v = *reinterpret_cast<const float2*>(dst + swz(g + 8 * h8, 8 * nt + 2 * q));
            G[nt][2 * h8] = v.x + (G[nt][2 * h8] + a[nt][2 * h8]);
            G[nt][2 * h8 + 1] = v.y + (G[nt][2 * h8 + 1] + a[nt][2 * h8 + 1]);
        }
}

// The per-token scalars of a backward stage (F = c alpha M + dv I); for the
// Cayley map F itself, formed over the stage's slices (stage_cayley in rounds
// of 4 tokens: the slots beyond the stage's 2 are never live and only read
// slot 0), with the scalars (1, 0).
template <bool Cay>
__device__ __forceinline__ void stage_scalars_or_cayley(const KParams& p, float2* cd, float* xs, unsigned live,
                                                        int lane, uint32_t* status)
{
    if constexpr (Cay) {
        stage_cayley<4>(p.alpha, xs, live, lane);
        if (lane < BST) cd[lane] = make_float2(1.0f, 0.0f);
        __syncwarp();
    } else {
        stage_scalars<BST>(p, cd, xs, live, lane, status);
    }
}

// Local pass: per chunk the gradient at t0 with nothing entering from the
// right (gloc) and W - I (Wq; zero for the last chunk of a sequence).  Cay:
// the Cayley map, its own instantiation (the elimination's registers would
// otherwise cost the other modes a CTA per SM), capped for three CTAs per SM
// (153 registers, no spills).
template <bool Cay>
__global__ void __launch_bounds__(BWARPS * 32, Cay ? 3 : 2)
k16b_local(KParams p, const float* __restrict__ x, const float* __restrict__ dS, float* __restrict__ gloc,
           float* __restrict__ Wq, uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    BSmem<false>& sm = reinterpret_cast<BSmem<false>*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * BWARPS + warp, stride = (int64_t)gridDim.x * BWARPS;
    const int64_t tok = p.H * NN;
    const int g = lane >> 2, q = lane & 3;
    const float m0 = (g == 2 * q) ? 1.0f : 0.0f, m1 = (g == 2 * q + 1) ? 1.0f : 0.0f;
    BFeed<false> feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = tok;
    feed.set(p);
#pragma unroll
    for (int s = 0; s < BNS - 1; ++s) feed.issue(sm, s, lane, p, x, nullptr, dS);
    int cs = 0, ps = BNS - 1;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        const int64_t base = (c.b * p.L * p.H + c.h) * NN;
        const bool more = c.tend < p.L;
        float G[2][4], Wt[2][4];
        load_acc(G, dS + base + (c.tend - 1) * tok, g, q);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) Wt[nt][i] = 0.0f;
        const int64_t hi = more ? c.tend : c.tend - 1, lo = c.tbeg + 1;
        for (int64_t ts = hi; ts >= lo; ts -= BST) {
            feed.issue(sm, ps, lane, p, x, nullptr, dS);
            ps = (ps + 1 == BNS) ? 0 : ps + 1;
            cp_async_wait<BNS - 1>();
            __syncwarp();
            const int nt = (ts - lo + 1 < BST) ? (int)(ts - lo + 1) : BST;
            stage_scalars_or_cayley<Cay>(p, sm.cd, sm.x[cs], (1u << nt) - 1u, lane, status);
#pragma unroll
            for (int j = 0; j < BST; ++j) {
                if (j < nt) {
                    const int64_t tau = ts - j;
                    const float2 cdj = sm.cd[j];
                    FragF ft;
                    make_frag_ft(sm.x[cs] + j * NN, cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, ft, more);
                    if (tau == c.tend) {
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) Wt[n2][i] = ft.fd[n2][i];     // W^T = F_{t1}^T
                    } else {
                        float a[2][4];
                        chain_product<true>(G, ft, a);
                        add_ds(sm.ds[cs] + j * NN, a, G, g, q);
                        if (more) {
                            chain_product<false>(Wt, ft, a);                       // F^T + W^T F^T
#pragma unroll
                            for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                                for (int i = 0; i < 4; ++i) Wt[n2][i] += a[n2][i];
                        }
                    }
                }
            }
            __syncwarp();
            cs = (cs + 1 == BNS) ? 0 : cs + 1;
        }
        // the chunk-gradient scan indexes chunks sequence-major: (b H + h) K + k
        const int64_t wchain = (c.b * p.H + c.h) * p.K + c.k;
        store_d(gloc + wchain * NN, G, g, q);
        float* w = Wq + wchain * NN;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {                 // W = (W^T)^T
                w[(8 * nt + 2 * q) * N + g + 8 * h8] = Wt[nt][2 * h8];
                w[(8 * nt + 2 * q + 1) * N + g + 8 * h8] = Wt[nt][2 * h8 + 1];
            }
    }
}

// Apply pass: per chunk G from the gradient entering from the right (Gin)
// down to t0, every dL/dx_t, and dL/dS0 from the first chunk.
template <bool Cay>
__global__ void __launch_bounds__(BWARPS * 32, 3)
k16b_apply(KParams p, const float* __restrict__ x, const float* __restrict__ S0, const float* __restrict__ S_fwd,
           const float* __restrict__ dS, const float* __restrict__ Gin, float* __restrict__ dx,
           float* __restrict__ dS0, uint32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    BSmem<true>& sm = reinterpret_cast<BSmem<true>*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * BWARPS + warp, stride = (int64_t)gridDim.x * BWARPS;
    const int64_t tok = p.H * NN;
    const int g = lane >> 2, q = lane & 3;
    const float m0 = (g == 2 * q) ? 1.0f : 0.0f, m1 = (g == 2 * q + 1) ? 1.0f : 0.0f;
    const bool detnorm = p.mode == MRU_MODE_DETNORM;
    constexpr bool cayley = Cay;
    BFeed<true> feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = tok;
    feed.set(p);
#pragma unroll
    for (int s = 0; s < BNS - 1; ++s) feed.issue(sm, s, lane, p, x, S_fwd, dS);
    int cs = 0, ps = BNS - 1;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        const int64_t seq = c.b * p.H + c.h;
        const int64_t base = (c.b * p.L * p.H + c.h) * NN;
        const bool boundary = c.tend < p.L;
        float G[2][4];
        if (boundary) load_acc(G, Gin + (seq * p.K + c.k) * NN, g, q);   // sequence-major chunk index
        else load_acc(G, dS + base + (c.tend - 1) * tok, g, q);
        const int64_t hi = boundary ? c.tend : c.tend - 1, lo = c.tbeg;
        for (int64_t ts = hi; ts >= lo; ts -= BST) {
            feed.issue(sm, ps, lane, p, x, S_fwd, dS);
            ps = (ps + 1 == BNS) ? 0 : ps + 1;
            cp_async_wait<BNS - 1>();
            __syncwarp();
            const int nt = (ts - lo + 1 < BST) ? (int)(ts - lo + 1) : BST;
            stage_scalars_or_cayley<Cay>(p, sm.cd, sm.x[cs], (1u << nt) - 1u, lane, status);
#pragma unroll
            for (int j = 0; j < BST; ++j) {
                if (j < nt) {
                    const int64_t tau = ts - j;
                    const float* xs = sm.x[cs] + j * NN;
                    const float2 cdj = sm.cd[j];
                    FragF ft;
                    make_frag_ft(xs, cdj.x, m0 * cdj.y, m1 * cdj.y, g, q, ft, false);
                    float a[2][4];
                    if (tau == c.tend) {                       // G_{t1-1} = dS_{t1-1} + Gin X_{t1}^T
                        chain_product<true>(G, ft, a);
                        add_ds(sm.ds[cs] + j * NN, a, G, g, q);
                        continue;
                    }
                    // dX = S_{t-1}^T G (S_{-1} = S0 or I)
                    float dX[2][4];
                    stage_acc(sm.stg, G, g, q);
                    __syncwarp();
                    if (tau >= 1) {
                        st_times_g(sm.s[cs] + j * NN, sm.stg, g, q, dX);
                    } else if (S0) {
                        float* s0t = sm.s[cs] + j * NN;    // S0 into the (unused) S tile of this token
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int gr = lane + 32 * i, row = gr >> 2, c4 = gr & 3;
                            *reinterpret_cast<float4*>(s0t + swz(row, 4 * c4)) =
                                *reinterpret_cast<const float4*>(S0 + seq * NN + row * N + 4 * c4);
                        }
                        __syncwarp();
                        st_times_g(s0t, sm.stg, g, q, dX);
                    } else {
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) dX[n2][i] = G[n2][i];
                    }
                    __syncwarp();
                    // the construction's chain rule
                    float out[2][4];
                    if constexpr (cayley) {
                        // X = 2 W^-1 - I, W = I - A, A = alpha (M - M^T) / 2: with
                        // W^-1 = I + F / 2, dA = 2 W^-T dX W^-T = 2 T + T F^T for
                        // T = dX + F^T dX / 2 (xs holds F), dM = alpha (dA - dA^T) / 2
                        stage_acc(sm.stg, dX, g, q);
                        __syncwarp();
                        float T[2][4], a2[2][4];
                        st_times_g(xs, sm.stg, g, q, T);      // F^T dX
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) T[n2][i] = fmaf(0.5f, T[n2][i], dX[n2][i]);
                        chain_product<true>(T, ft, a2);       // T F^T
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) a2[n2][i] = fmaf(2.0f, T[n2][i], a2[n2][i]);   // dA
                        __syncwarp();
                        stage_acc(sm.stg, a2, g, q);
                        __syncwarp();
                        const float ha = 0.5f * p.alpha;
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int h8 = 0; h8 < 2; ++h8)
#pragma unroll
                                for (int e = 0; e < 2; ++e)
                                    out[n2][2 * h8 + e] =
                                        ha * (a2[n2][2 * h8 + e] - sm.stg[swz(8 * n2 + 2 * q + e, g + 8 * h8)]);
                        __syncwarp();
                    } else if (!detnorm) {
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) out[n2][i] = p.alpha * dX[n2][i];
                    } else {
                        // <dX, Xr> with Xr = I + alpha M at the accumulator positions
                        float part = 0.0f;
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int h8 = 0; h8 < 2; ++h8) {
                                const float2 v = *reinterpret_cast<const float2*>(xs + swz(g + 8 * h8, 8 * n2 + 2 * q));
                                part = fmaf(dX[n2][2 * h8], fmaf(p.alpha, v.x, h8 == n2 ? m0 : 0.0f), part);
                                part = fmaf(dX[n2][2 * h8 + 1], fmaf(p.alpha, v.y, h8 == n2 ? m1 : 0.0f), part);
                            }
                        const float s = warp_sum(part) * (1.0f / N);
                        FragF fe;
                        make_frag_ft(xs, p.alpha, 0.0f, 0.0f, g, q, fe, true);
                        float f2 = 0.0f;
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int i = 0; i < 4; ++i) f2 = fmaf(fe.fd[n2][i], fe.fd[n2][i], f2);
                        const float fro2 = warp_sum(f2);
                        float Z[2][4];
                        if (fro2 <= 0.8f) inverse_t_ns(fe, fro2, sm.stg, g, q, Z);
                        else inverse_t_pivoted(xs, p.alpha, sm.stg, lane, Z);
                        const float c1 = 1.0f + cdj.y;       // c (dv = c - 1)
                        const float ac = cdj.x == 0.0f ? 0.0f : p.alpha * c1;   // singular token: zero
#pragma unroll
                        for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                            for (int h8 = 0; h8 < 2; ++h8) {
                                const float i0 = h8 == n2 ? m0 : 0.0f, i1 = h8 == n2 ? m1 : 0.0f;
                                out[n2][2 * h8] = ac * fmaf(-s, Z[n2][2 * h8] + i0, dX[n2][2 * h8]);
                                out[n2][2 * h8 + 1] = ac * fmaf(-s, Z[n2][2 * h8 + 1] + i1, dX[n2][2 * h8 + 1]);
                            }
                    }
                    store_d(dx + base + tau * tok, out, g, q);
                    // G_{t-1} = dS_{t-1} + G X_t^T, or dS0 = G X_1^T at the first token
                    if (tau > lo || tau == 0) {
                        chain_product<true>(G, ft, a);
                        if (tau == 0) {
                            if (dS0) {
#pragma unroll
                                for (int n2 = 0; n2 < 2; ++n2)
#pragma unroll
                                    for (int i = 0; i < 4; ++i) a[n2][i] += G[n2][i];
                                store_d(dS0 + seq * NN, a, g, q);
                            }
                        } else {
                            add_ds(sm.ds[cs] + j * NN, a, G, g, q);
                        }
                    }
                }
            }
            __syncwarp();
            cs = (cs + 1 == BNS) ? 0 : cs + 1;
        }
    }
}

// CTAs of a persistent launch: resident CTAs per SM times the SM count,
// cached per device and kernel slot (one slot per kernel instantiation:
// reduce 0, 1, 6, 11; apply 2, 3, 7, 8, 12, 13, 14; backward 4, 5, and 16, 17
// for the Cayley map; single-read 9, 10, 15); no more than the chains need.
constexpr int kSlots = 18;
std::atomic<int> g_resident[64][kSlots];

// The orthogonal construction the passes apply to each slice: 0 none, 1 the
// Cayley map, 2 the exponential map.
int transform_of(const KParams& p)
{
    return p.mode == MRU_MODE_CAYLEY ? 1 : p.mode == MRU_MODE_EXPM ? 2 : 0;
}

cudaError_t persistent_grid(int slot, const void* kern, int threads, size_t smem, int warps, int64_t nchains,
                            unsigned& grid)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (slot < 0 || slot >= kSlots) return cudaErrorInvalidValue;
    int res = (dev >= 0 && dev < 64) ? g_resident[dev][slot].load(std::memory_order_relaxed) : 0;
    if (res <= 0) {
        int sms = 0, per_sm = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem)) != cudaSuccess)
            return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        res = sms * per_sm;
        if (dev >= 0 && dev < 64) g_resident[dev][slot].store(res, std::memory_order_relaxed);
    }
    const int64_t need = (nchains + warps - 1) / warps;
    grid = (unsigned)(need < res ? need : res);
    return cudaSuccess;
}

}  // namespace

bool supports(const KParams& p, bool readout)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_F32 && !readout &&
           (p.mode == MRU_MODE_RESHAPE || p.mode == MRU_MODE_DETNORM || p.mode == MRU_MODE_CAYLEY ||
            p.mode == MRU_MODE_EXPM) &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_TF32X3) && p.chunk > 0 && p.chunk % kSub == 0;
}

// Chunk length: 8 m tokens, m a power of two (at most 16) that keeps at
// least 8192 chains when the workload allows (about three per warp of a full
// persistent grid), so that long sequences get long chunks (few chunk
// totals, little carry work per token).  Measured on B200: 32 tokens for
// 262,144 token-heads, 128 for 2,097,152.
int32_t preferred_chunk(int64_t token_heads)
{
    int32_t m = 1;
    while (m < 16 && token_heads / ((int64_t)kSub * 2 * m) >= 8192) m *= 2;
    return kSub * m;
}

// Levels of the carry scan for nseq sequences of K chunk totals, laid out
// from byte offset off.  G = 16 unless K > 16^4 (then the smallest power of
// two with G^4 >= K), so that at most three levels sit below the top.
CarryPlan carry_plan(int64_t nseq, int64_t K, size_t off)
{
    CarryPlan cp;
    memset(&cp, 0, sizeof cp);
    cp.nseq = nseq;
    cp.gshift = 4;
    while (((int64_t)1 << (4 * cp.gshift)) < K) ++cp.gshift;
    cp.G = 1 << cp.gshift;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) / 256 * 256;
        return o;
    };
    cp.cnt[0] = K;
    int l = 0;
    while (cp.cnt[l] > cp.G) {
        cp.cnt[l + 1] = (cp.cnt[l] + cp.G - 1) / cp.G;
        cp.R[l] = take((size_t)nseq * cp.cnt[l] * NN * (l == 0 ? sizeof(float) : sizeof(double)));
        cp.Tot[l] = take((size_t)nseq * cp.cnt[l + 1] * NN * sizeof(double));
        ++l;
    }
    cp.levels = l;
    cp.Etop = take((size_t)nseq * cp.cnt[l] * NN * sizeof(double));
    cp.ctr_begin = off;
    for (int i = 0; i < l; ++i) cp.ctr[i] = take((size_t)nseq * cp.cnt[i + 1] * sizeof(unsigned));
    cp.ctr[l] = take((size_t)nseq * sizeof(unsigned));
    cp.ctr_bytes = off - cp.ctr_begin;
    cp.end = off;
    return cp;
}

cudaError_t launch_reduce(const KParams& p, const float* x, float* totals, const CarryPlan& cp, char* ws,
                          uint32_t* status, float* fout, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(RSmem) * RWARPS;
    const bool per_token = p.mode == MRU_MODE_DETNORM && !p.add_identity;
    const int tr = transform_of(p);
    auto kern = tr == 1 ? k16_reduce<false, 1> : tr == 2 ? k16_reduce<false, 2>
                        : per_token ? k16_reduce<true> : k16_reduce<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    if ((e = persistent_grid(tr == 1 ? 6 : tr == 2 ? 11 : per_token ? 1 : 0, (const void*)kern, RWARPS * 32, sm,
                             RWARPS, nchains,
                             grid)) !=
        cudaSuccess)
        return e;
    kern<<<grid, RWARPS * 32, sm, s>>>(p, x, totals, reinterpret_cast<unsigned*>(ws + cp.ctr_begin),
                                       (int64_t)(cp.ctr_bytes / sizeof(unsigned)), status, tr != 0 ? fout : nullptr);
    return cudaGetLastError();
}

cudaError_t launch_carry(const KParams& p, const float* totals, const CarryPlan& cp, char* ws, const float* S0,
                         cudaStream_t s)
{
    const int64_t units = cp.nseq * (cp.levels > 0 ? cp.cnt[1] : 1);
    if (p.B * p.H * p.K == 0 || units == 0) return cudaSuccess;
    const size_t sm = sizeof(CSmem) * CWARPS;
    cudaError_t e = cudaFuncSetAttribute(k16_carry, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k16_carry<<<(unsigned)((units + CWARPS - 1) / CWARPS), CWARPS * 32, sm, s>>>(p, totals, cp, ws, S0);
    return cudaGetLastError();
}

// Chunk totals, in-group prefixes, group aggregates, carries and inclusive
// prefixes, per-token scalars, then the control block, laid out from byte
// offset off.  Groups of 16 chunks, or the smallest power of two with at
// most 4096 groups per sequence (the look-back multiplies one aggregate per
// group it passes; fewer, longer groups keep that chain short).
FusedPlan fused_plan(const KParams& p, size_t off)
{
    FusedPlan fp;
    memset(&fp, 0, sizeof fp);
    const int64_t nseq = p.B * p.H;
    fp.gshift = 4;
    while (p.K > ((int64_t)4096 << fp.gshift) && fp.gshift < 10) ++fp.gshift;
    fp.NG = p.K > 0 ? (p.K + (1 << fp.gshift) - 1) >> fp.gshift : 0;
    fp.Lp = (p.L + 7) / 8 * 8;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) / 256 * 256;
        return o;
    };
    fp.tot = take((size_t)nseq * p.K * NN * sizeof(float));
    fp.R0 = take((size_t)nseq * p.K * NN * sizeof(float));
    fp.agg = take((size_t)nseq * fp.NG * NN * sizeof(double));
    fp.incl = take((size_t)nseq * fp.NG * NN * sizeof(double));
    fp.excl = take((size_t)nseq * fp.NG * NN * sizeof(float));
    fp.cd = take(p.mode == MRU_MODE_DETNORM ? (size_t)nseq * fp.Lp * sizeof(float2) : 0);
    fp.ctl = off;
    fp.gcnt = fp.ctl + 16;
    fp.gflag = fp.gcnt + (size_t)nseq * fp.NG * sizeof(unsigned);
    take(16 + 2 * (size_t)nseq * fp.NG * sizeof(unsigned));
    fp.ctl_bytes = off - fp.ctl;
    fp.end = off;
    return fp;
}

namespace {
std::atomic<int32_t> g_stall_ms{0};

// Reduce items handed out before the first apply item: about 64 MB of
// embeddings between a chain's reduce and its apply (measured on B200 for
// B8 H8 L4096 with 32-token chunks: 16 MB 0.49 ms, 32 MB 0.45, 64 MB 0.38),
// and at least a group of chains of every head plus one row of heads, which
// the waits need (see fused_decode).
int64_t fused_lead(const KParams& p, const FusedPlan& fp)
{
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t chain_bytes = (int64_t)p.chunk * NN * (int64_t)sizeof(float);
    int64_t lead = ((int64_t)64 << 20) / (chain_bytes > 0 ? chain_bytes : 1);
    const int64_t need = ((int64_t)1 << fp.gshift) * p.H + p.H;
    if (lead < need) lead = need;
    return lead < nchains ? lead : nchains;
}
}

void set_stall_test(int32_t ms) { g_stall_ms.store(ms, std::memory_order_relaxed); }

cudaError_t launch_fused(const KParams& p, const FusedPlan& fp, char* ws, const float* x, const float* S0,
                         float* S_out, uint32_t* status, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    FCtl f;
    f.ctr = reinterpret_cast<unsigned*>(ws + fp.ctl);
    f.gcnt = reinterpret_cast<unsigned*>(ws + fp.gcnt);
    f.gflag = reinterpret_cast<unsigned*>(ws + fp.gflag);
    f.tot = reinterpret_cast<float*>(ws + fp.tot);
    f.R0 = reinterpret_cast<float*>(ws + fp.R0);
    f.agg = reinterpret_cast<double*>(ws + fp.agg);
    f.incl = reinterpret_cast<double*>(ws + fp.incl);
    f.excl = reinterpret_cast<float*>(ws + fp.excl);
    f.cd = reinterpret_cast<float2*>(ws + fp.cd);
    f.Lp = fp.Lp;
    f.NG = fp.NG;
    f.gshift = fp.gshift;
    f.lead = fused_lead(p, fp);
    const int32_t stall = g_stall_ms.exchange(0, std::memory_order_relaxed);
    f.stall_first = stall > 0;
    f.limit_ns = stall > 0 ? (uint64_t)stall * 1000000ull : 2000000000ull;     // 2 s unless testing
    cudaError_t e = cudaMemsetAsync(ws + fp.ctl, 0, fp.ctl_bytes, s);
    if (e != cudaSuccess) return e;
    const int tr = transform_of(p);
    auto kern = tr == 1 ? k16_fused<1> : tr == 2 ? k16_fused<2> : k16_fused<0>;
    const size_t sm = sizeof(FSmem) * FWARPS;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess)
        return e;
    unsigned grid = 0;
    if ((e = persistent_grid(tr == 2 ? 15 : 9 + tr, (const void*)kern, FWARPS * 32, sm, FWARPS, nchains, grid)) !=
        cudaSuccess)
        return e;
    kern<<<grid, FWARPS * 32, sm, s>>>(p, f, x, S0, S_out, status);
    return cudaGetLastError();
}

bool supports_backward(const KParams& p)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_F32 &&
           (p.mode == MRU_MODE_RESHAPE || (p.mode == MRU_MODE_DETNORM && p.add_identity) ||
            p.mode == MRU_MODE_CAYLEY) &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_TF32X3) && p.chunk > 0;
}

cudaError_t launch_bwd_local(const KParams& p, const float* x, const float* dS, float* gloc, float* Wq,
                             uint32_t* status, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(BSmem<false>) * BWARPS;
    const bool cay = p.mode == MRU_MODE_CAYLEY;
    auto kern = cay ? k16b_local<true> : k16b_local<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    if ((e = persistent_grid(cay ? 16 : 4, (const void*)kern, BWARPS * 32, sm, BWARPS, nchains, grid)) != cudaSuccess)
        return e;
    kern<<<grid, BWARPS * 32, sm, s>>>(p, x, dS, gloc, Wq, status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_apply(const KParams& p, const float* x, const float* S0, const float* S_fwd, const float* dS,
                             const float* Gin, float* dx, float* dS0, uint32_t* status, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(BSmem<true>) * BWARPS;
    const bool cay = p.mode == MRU_MODE_CAYLEY;
    auto kern = cay ? k16b_apply<true> : k16b_apply<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    if ((e = persistent_grid(cay ? 17 : 5, (const void*)kern, BWARPS * 32, sm, BWARPS, nchains, grid)) != cudaSuccess)
        return e;
    kern<<<grid, BWARPS * 32, sm, s>>>(p, x, S0, S_fwd, dS, Gin, dx, dS0, status);
    return cudaGetLastError();
}

cudaError_t launch_apply(const KParams& p, const float* x, const CarryPlan& cp, const char* ws, float* S_out,
                         uint32_t* status, const float* S0, bool direct, bool pre_transformed, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(ASmem) * AWARPS;
    const int tr = pre_transformed && !direct ? 3 : transform_of(p);
    auto kern = tr == 1   ? (direct ? k16_apply<true, 1> : k16_apply<false, 1>)
                : tr == 2 ? (direct ? k16_apply<true, 2> : k16_apply<false, 2>)
                : tr == 3 ? k16_apply<false, 3>
                          : (direct ? k16_apply<true> : k16_apply<false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    const int slot = tr == 1 ? (direct ? 8 : 7) : tr == 2 ? (direct ? 13 : 12) : tr == 3 ? 14 : (direct ? 3 : 2);
    if ((e = persistent_grid(slot, (const void*)kern, AWARPS * 32, sm, AWARPS,
                             nchains, grid)) !=
        cudaSuccess)
        return e;
    kern<<<grid, AWARPS * 32, sm, s>>>(p, x, cp, ws, S_out, status, direct ? S0 : nullptr);
    return cudaGetLastError();
}

}  // namespace n16
}  // namespace mru
