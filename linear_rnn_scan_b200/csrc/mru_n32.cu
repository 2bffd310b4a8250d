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
#include <type_traits>

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

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* smem_row)
{
    const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(smem_row));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
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
// PK: the residual by one packed subtraction (same values).
template <bool PK = true>
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo)
{
    hi = pack_bf16(x0, x1);
    if (PK) {
        float r0, r1;
        f2::up(f2::sub(f2::pk(x0, x1), f2::pk(bf16_lo(hi), bf16_hi(hi))), r0, r1);
        lo = pack_bf16(r0, r1);
    } else {
        lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
    }
}

// The state: 32 x 32 fp32 in accumulator layout, st[mt][nt][i] holds
// element (16 mt + g + 8 (i >> 1), 8 nt + 2 q + (i & 1)).
using State = float[2][4][4];

// A fragments (hi, lo) of the state: the accumulator tile (mt, 2 kt) and
// (mt, 2 kt + 1) are exactly the A fragment (mt, kt) of m16n8k16.
template <bool PK = true>
__device__ __forceinline__ void state_frags(const State& st, uint32_t (&ah)[2][2][4], uint32_t (&al)[2][2][4])
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            split_pair<PK>(st[mt][2 * kt][0], st[mt][2 * kt][1], ah[mt][kt][0], al[mt][kt][0]);
            split_pair<PK>(st[mt][2 * kt][2], st[mt][2 * kt][3], ah[mt][kt][1], al[mt][kt][1]);
            split_pair<PK>(st[mt][2 * kt + 1][0], st[mt][2 * kt + 1][1], ah[mt][kt][2], al[mt][kt][2]);
            split_pair<PK>(st[mt][2 * kt + 1][2], st[mt][2 * kt + 1][3], ah[mt][kt][3], al[mt][kt][3]);
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

// B fragments of M^T (B[k][n] = M[n][k]) for all (kt, nt), in the layout of
// load_m_frags: bm[kt][nt][h] holds M[8 nt + g][16 kt + 8 h + 2 q], + 1
// (ldmatrix without transposition on rows of M).
__device__ __forceinline__ void load_mt_frags(const unsigned char* xs, int lane, uint32_t (&bm)[2][4][2])
{
    const int r = lane & 7, kh = (lane >> 3) & 1, np2 = lane >> 4;
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t v[4];
            ldsm_x4(v, xs + (8 * (2 * np + np2) + r) * ROWB + (16 * kt + 8 * kh) * 2);
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
    // k - n = c + d (+ 1) with |d| <= 7 and c a multiple of 8: off the
    // diagonal 8 x 8 blocks every entry of the register has the sign of c
    // (c is a compile-time constant at every use, so these fold away)
    if (c >= 8) return lower ? v : 0u;
    if (c <= -8) return lower ? 0u : v;
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

// Three-term split of a pair (x ~ hi + mid + lo, the residual below 2^-26 |x|).
__device__ __forceinline__ void split_pair3(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo)
{
    hi = pack_bf16(x0, x1);
    const uint64_t r = f2::sub(f2::pk(x0, x1), f2::pk(bf16_lo(hi), bf16_hi(hi)));
    float r0, r1;
    f2::up(r, r0, r1);
    mid = pack_bf16(r0, r1);
    f2::up(f2::sub(r, f2::pk(bf16_lo(mid), bf16_hi(mid))), r0, r1);
    lo = pack_bf16(r0, r1);
}

// A fragments (hi, mid, lo) of the state, as state_frags.
__device__ __forceinline__ void state_frags3(const State& st, uint32_t (&ah)[2][2][4], uint32_t (&am)[2][2][4],
                                             uint32_t (&al)[2][2][4])
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            split_pair3(st[mt][2 * kt][0], st[mt][2 * kt][1], ah[mt][kt][0], am[mt][kt][0], al[mt][kt][0]);
            split_pair3(st[mt][2 * kt][2], st[mt][2 * kt][3], ah[mt][kt][1], am[mt][kt][1], al[mt][kt][1]);
            split_pair3(st[mt][2 * kt + 1][0], st[mt][2 * kt + 1][1], ah[mt][kt][2], am[mt][kt][2], al[mt][kt][2]);
            split_pair3(st[mt][2 * kt + 1][2], st[mt][2 * kt + 1][3], ah[mt][kt][3], am[mt][kt][3], al[mt][kt][3]);
        }
}

// tri_product with the state in three terms (smallest first).
template <bool LOWER>
__device__ __forceinline__ void tri_product3(const uint32_t (&ah)[2][2][4], const uint32_t (&am)[2][2][4],
                                             const uint32_t (&al)[2][2][4], const uint32_t (&bm)[2][4][2], int d,
                                             State& acc)
{
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            if (LOWER && 16 * kt + 15 <= 8 * nt) continue;
            if (!LOWER && 16 * kt >= 8 * nt + 7) continue;
            const bool first = kt == 0 || (LOWER ? 15 <= 8 * nt : 0 >= 8 * nt + 7);
            const uint32_t b0 = tri_mask(bm[kt][nt][0], 16 * kt - 8 * nt, d, LOWER);
            const uint32_t b1 = tri_mask(bm[kt][nt][1], 16 * kt + 8 - 8 * nt, d, LOWER);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                if (first) mma_bf16_first(acc[mt][nt], al[mt][kt], b0, b1);
                else mma_bf16(acc[mt][nt], al[mt][kt], b0, b1);
                mma_bf16(acc[mt][nt], am[mt][kt], b0, b1);
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

// M^T at this lane's accumulator positions: element (16 mt + g + 8 h,
// 8 nt + 2 q + s) of M^T is M[8 nt + 2 q + s][16 mt + g + 8 h].
__device__ __forceinline__ void load_mt_d(const unsigned char* xs, int g, int q, float (&md)[2][4][4])
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 8 * nt + 2 * q + (i & 1), col = 16 * mt + g + 8 * (i >> 1);
                const uint16_t v = *reinterpret_cast<const uint16_t*>(xs + row * ROWB + col * 2);
                md[mt][nt][i] = __uint_as_float((uint32_t)v << 16);
            }
}

// One token applied to the state, from the factor fragments bm (M for
// state X, M^T for state X^T = U^T D L^T: the lower mask then picks U_s^T,
// the upper one L_s^T) and the same matrix at the accumulator positions md.
// split: state is Q = P - I and the factors' identity parts enter as the
// extra terms; otherwise the state is the full product.
template <bool SPLIT, int TERMS = 2>
__device__ __forceinline__ void apply_token_f(State& st, const uint32_t (&bm)[2][4][2], const float (&md)[2][4][4],
                                              const float* Dv, const float* Dm1, float a, int lane)
{
    const int g = lane >> 2, q = lane & 3, d = 2 * q - g;
    constexpr bool PK = SPLIT || TERMS == 3;
    uint32_t ah[2][2][4], al[2][2][4];
    State acc;
    auto product = [&](auto lower_tag) {
        constexpr bool LOWER = decltype(lower_tag)::value;
        if constexpr (TERMS == 3) {
            uint32_t am[2][2][4];
            state_frags3(st, ah, am, al);
            tri_product3<LOWER>(ah, am, al, bm, d, acc);
        } else {
            state_frags<PK>(st, ah, al);
            tri_product<LOWER>(ah, al, bm, d, acc);
        }
    };
    // The element updates run on packed pairs (columns 2 q, 2 q + 1 of a
    // row), with the scalar rounding of every operation: fewer issue slots
    // for the split-form reduce chain and the backward's three-term chains;
    // the forward apply pass, bound by memory, keeps the scalar form
    // (measured on B200: packed there made it 4 % slower).
    const uint64_t a2 = f2::pk(a, a);
    auto update = [&](auto lower_tag) {
        constexpr bool LOWER = decltype(lower_tag)::value;
        if constexpr (!PK) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) st[mt][nt][i] += a * acc[mt][nt][i];
            return;
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // 8 x 8 block (2 mt + h, nt): below, above or on the diagonal
                    const int R = 2 * mt + h;
                    float t[2];
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        const int cs = 2 * q + s2;
                        const float m = md[mt][nt][2 * h + s2];
                        t[s2] = LOWER ? (R > nt ? m : R < nt ? 0.0f : (g > cs ? m : 0.0f))
                                      : (R < nt ? m : R > nt ? 0.0f : (g < cs ? m : 0.0f));
                    }
                    const uint64_t ac = f2::pk(acc[mt][nt][2 * h], acc[mt][nt][2 * h + 1]);
                    const uint64_t sv = f2::pk(st[mt][nt][2 * h], st[mt][nt][2 * h + 1]);
                    f2::up(f2::fma(a2, SPLIT ? f2::add(f2::pk(t[0], t[1]), ac) : ac, sv), st[mt][nt][2 * h],
                           st[mt][nt][2 * h + 1]);
                }
    };
    // --- P L ---
    product(std::true_type{});
    update(std::true_type{});
    // --- (P L) D ---
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const float2 dv = *reinterpret_cast<const float2*>(Dv + 8 * nt + 2 * q);
        const float2 dm = *reinterpret_cast<const float2*>(Dm1 + 8 * nt + 2 * q);
        const uint64_t dv2 = f2::pk(dv.x, dv.y);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int R = 2 * mt + h;
                float v0, v1;
                if (PK) {
                    f2::up(f2::mul(f2::pk(st[mt][nt][2 * h], st[mt][nt][2 * h + 1]), dv2), v0, v1);
                } else {
                    v0 = st[mt][nt][2 * h] * dv.x;
                    v1 = st[mt][nt][2 * h + 1] * dv.y;
                }
                if (SPLIT && R == nt && g == 2 * q) v0 += dm.x;
                if (SPLIT && R == nt && g == 2 * q + 1) v1 += dm.y;
                st[mt][nt][2 * h] = v0;
                st[mt][nt][2 * h + 1] = v1;
            }
    }
    // --- (P L D) U ---
    product(std::false_type{});
    update(std::false_type{});
}

// One token applied to the state (forward: the state times X = L D U).
template <bool SPLIT>
__device__ __forceinline__ void apply_token(State& st, const unsigned char* xs, const float* Dv, const float* Dm1,
                                            float a, int lane)
{
    uint32_t bm[2][4][2];
    load_m_frags(xs, lane, bm);
    float md[2][4][4];
    load_m_d(xs, lane >> 2, lane & 3, md);
    apply_token_f<SPLIT>(st, bm, md, Dv, Dm1, a, lane);
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

// ---- backward (vector-Jacobian product) on the tensor cores ----------------
//
// G_t = dL/dS_t (later states included): G_{t-1} = dS_{t-1} + G_t X_t^T and
// dL/dX_t = S_{t-1}^T G_t (the chain rule of S_t = S_{t-1} X_t), chunked as
// the n = 16 backward: a local pass per chunk [t0, t1) (the gradient at t0
// with nothing entering from the right, and W - I with W = X_{t0+1} ...
// X_{t1}), the generic fp64 right-to-left scan of the chunk gradients, and an
// apply pass (G from the gradient entering from the right down to t0, dX_t,
// the LDU chain rule).  Right products by X^T = U^T D L^T run as the
// forward's factor steps with the fragments of M^T (apply_token_f); W is
// carried as W^T so that its left multiplications become right ones.  The
// tokens of a chunk stream in reverse order, one per stage: x_t (bf16), and
// for the apply pass S_{t-1}, and dS_{t-1} (fp32, rows padded so that the
// fragment reads are free of bank conflicts).
//
// dX = S^T G is a full product in split bf16 (S^T hi, lo times G hi, lo, the
// lo lo term dropped), G's halves staged in shared memory for ldmatrix.trans.
// Chain rule of X = L D U (L = I + a Ls, U = I + a Us, D_i = exp(d tanh M_ii)):
//   dM_ij = a D_j (dX U^T)_ij      (i > j;  dX U^T = dX + a dX Us^T)
//   dM_ij = a D_i (L^T dX)_ij      (i < j;  L^T dX = dX + a Ls^T dX)
//   dM_ii = D_i d (1 - tanh^2 M_ii) (L^T dX U^T)_ii,
//           (L^T dX U^T)_ii = (L^T dX)_ii + a sum_{k > i} (L^T dX)_ik M_ik.

constexpr int SROW = 36;             // padded row stride (words) of a staged fp32 S_{t-1}
constexpr int DROW = 40;             // padded row stride (words) of a staged fp32 dS_{t-1}
constexpr int BLWARPS = 4;           // local pass: warps per CTA (2 CTAs per SM, 255 registers)
constexpr int BAWARPS = 2;           // apply pass: warps per CTA (4 CTAs per SM)

template <bool APPLY>
struct BSmem32 {
    unsigned char x[2][SLICEB];                      // x_t
    float ds[APPLY ? 1 : 2][N * DROW];               // dS_{t-1} (apply: one buffer, filled as its token starts)
    float s[APPLY ? 2 : 1][APPLY ? N * SROW : 4];    // S_{t-1}
    unsigned char stg[APPLY ? 3 : 1][APPLY ? SLICEB : 16];   // bf16 terms (hi, mid, lo) of a staged matrix
    float dd[2][3][N];                               // per stage: D_i, D_i - 1, d (1 - tanh^2 M_ii)
};

// D_i, D_i - 1 and dD_i / dM_ii / D_i of one token (lane i: diagonal entry i).
__device__ __forceinline__ void stage_dd_b(const KParams& p, const unsigned char* xs, float (&dd)[3][N], int lane)
{
    const uint16_t mb = *reinterpret_cast<const uint16_t*>(xs + lane * ROWB + lane * 2);
    const float th = tanhf(__uint_as_float((uint32_t)mb << 16));
    const float dm1 = expm1f(p.ldu_d * th);
    dd[0][lane] = 1.0f + dm1;
    dd[1][lane] = dm1;
    dd[2][lane] = p.ldu_d * fmaf(-th, th, 1.0f);
    __syncwarp();
}

// A 32 x 32 fp32 matrix in accumulator layout from rows `stride` words apart.
__device__ __forceinline__ void load_state(State& st, const float* src, int stride, int g, int q)
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 v = *reinterpret_cast<const float2*>(src + (16 * mt + g + 8 * h) * stride + 8 * nt + 2 * q);
                st[mt][nt][2 * h] = v.x;
                st[mt][nt][2 * h + 1] = v.y;
            }
}

// st += the matrix at src (rows `stride` words apart).
__device__ __forceinline__ void add_state(State& st, const float* src, int stride, int g, int q)
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 v = *reinterpret_cast<const float2*>(src + (16 * mt + g + 8 * h) * stride + 8 * nt + 2 * q);
                st[mt][nt][2 * h] += v.x;
                st[mt][nt][2 * h + 1] += v.y;
            }
}

// The producer side of a backward warp's pipeline: one token per stage, in
// reverse order along the warp's chains.  Local pass: tokens t1 (when a
// chunk follows) down to t0 + 1; apply pass: t1 (when a chunk follows, for
// the gradient entering from the right) down to t0.
template <bool APPLY>
struct BFeed32 {
    int64_t chain, stride, nchains, tok;
    int64_t tau, lo, base;

    __device__ __forceinline__ void set(const KParams& p)
    {
        for (; chain < nchains; chain += stride) {      // skips chains with nothing to stream
            const Chain c = chain_at(p, chain);
            base = (c.b * p.L * p.H + c.h) * NN;
            tau = c.tend < p.L ? c.tend : c.tend - 1;
            lo = APPLY ? c.tbeg : c.tbeg + 1;
            if (tau >= lo) return;
        }
    }
    __device__ __forceinline__ void issue(BSmem32<APPLY>& sm, int slot, int lane, const KParams& p,
                                          const uint16_t* x, const float* S_fwd, const float* dS)
    {
        if (chain < nchains) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {          // x_tau: 128 granules of 16 bytes
                const int gi = lane + 32 * i, row = gi >> 2, c4 = gi & 3;
                cp_async16(sm.x[slot] + row * ROWB + c4 * 16, x + base + tau * tok + row * N + c4 * 8);
            }
            if (tau >= 1) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {      // dS_{tau-1} (local pass) or S_{tau-1} (apply): 256 granules
                    const int gi = lane + 32 * i, row = gi >> 3, c4 = gi & 7;
                    if (APPLY)
                        cp_async16(&sm.s[slot][0] + row * SROW + 4 * c4,
                                   S_fwd + base + (tau - 1) * tok + row * N + 4 * c4);
                    else
                        cp_async16(sm.ds[slot] + row * DROW + 4 * c4, dS + base + (tau - 1) * tok + row * N + 4 * c4);
                }
            }
            if (--tau < lo) {
                chain += stride;
                set(p);
            }
        }
        cp_async_commit();
    }
};

// The chunk's chains are counted sequence-major by the chunk-gradient scan:
// (b H + h) K + k.
__device__ __forceinline__ int64_t seq_major(const KParams& p, const Chain& c)
{
    return (c.b * p.H + c.h) * p.K + c.k;
}

// Local pass: per chunk, G from dS_{t1-1} down to t0 (nothing entering from
// the right) and W^T = (X_{t0+1} ... X_{t1})^T - I.
__global__ void __launch_bounds__(BLWARPS * 32, 2)
k32b_local(KParams p, const uint16_t* __restrict__ x, const float* __restrict__ dS, float* __restrict__ gloc,
           float* __restrict__ Wq)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    BSmem32<false>& sm = reinterpret_cast<BSmem32<false>*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * BLWARPS + warp, stride = (int64_t)gridDim.x * BLWARPS;
    const int64_t tok = p.H * NN;
    const int g = lane >> 2, q = lane & 3;
    BFeed32<false> feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = tok;
    feed.set(p);
    feed.issue(sm, 0, lane, p, x, nullptr, dS);
    int cs = 0;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        const int64_t base = (c.b * p.L * p.H + c.h) * NN;
        const bool more = c.tend < p.L;
        State G, Wt;
        load_state(G, dS + base + (c.tend - 1) * tok, N, g, q);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) Wt[mt][nt][i] = 0.0f;
        const int64_t hi = more ? c.tend : c.tend - 1, lo = c.tbeg + 1;
        for (int64_t tau = hi; tau >= lo; --tau) {
            feed.issue(sm, cs ^ 1, lane, p, x, nullptr, dS);
            cp_async_wait<1>();
            __syncwarp();
            const unsigned char* xs = sm.x[cs];
            stage_dd_b(p, xs, sm.dd[cs], lane);
            uint32_t bm[2][4][2];
            load_mt_frags(xs, lane, bm);
            float md[2][4][4];
            load_mt_d(xs, g, q, md);
            if (more) apply_token_f<true, 3>(Wt, bm, md, sm.dd[cs][0], sm.dd[cs][1], p.ldu_a, lane);   // W^T X^T
            if (tau < c.tend) {                                     // G <- dS_{tau-1} + G X_tau^T
                apply_token_f<false, 3>(G, bm, md, sm.dd[cs][0], sm.dd[cs][1], p.ldu_a, lane);
                add_state(G, sm.ds[cs], DROW, g, q);
            }
            __syncwarp();
            cs ^= 1;
        }
        const int64_t wchain = seq_major(p, c);
        store_state(gloc + wchain * NN, G, g, q);
        float* w = Wq + wchain * NN;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {                   // W = (W^T)^T
                    const int row = 16 * mt + g + 8 * (i >> 1), col = 8 * nt + 2 * q + (i & 1);
                    w[col * N + row] = more ? Wt[mt][nt][i] : 0.0f;
                }
    }
}

// The bf16 halves (A fragments from state_frags) of a matrix written row-major
// into stg[0] (hi) and stg[1] (lo), rows padded to ROWB bytes.
__device__ __forceinline__ void stage_frags(unsigned char (*stg)[SLICEB], const uint32_t (&ah)[2][2][4],
                                            const uint32_t (&al)[2][2][4], int g, int q)
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int kt = 0; kt < 2; ++kt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 16 * mt + g + 8 * (i & 1), col = 16 * kt + 2 * q + 8 * (i >> 1);
                *reinterpret_cast<uint32_t*>(stg[0] + row * ROWB + col * 2) = ah[mt][kt][i];
                *reinterpret_cast<uint32_t*>(stg[1] + row * ROWB + col * 2) = al[mt][kt][i];
            }
}

// The three bf16 terms of a matrix (A fragments from state_frags3) written
// row-major into stg[0..2].
__device__ __forceinline__ void stage_frags3(unsigned char (*stg)[SLICEB], const uint32_t (&ah)[2][2][4],
                                             const uint32_t (&am)[2][2][4], const uint32_t (&al)[2][2][4], int g,
                                             int q)
{
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int kt = 0; kt < 2; ++kt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 16 * mt + g + 8 * (i & 1), col = 16 * kt + 2 * q + 8 * (i >> 1);
                *reinterpret_cast<uint32_t*>(stg[0] + row * ROWB + col * 2) = ah[mt][kt][i];
                *reinterpret_cast<uint32_t*>(stg[1] + row * ROWB + col * 2) = am[mt][kt][i];
                *reinterpret_cast<uint32_t*>(stg[2] + row * ROWB + col * 2) = al[mt][kt][i];
            }
}

// dX = S^T G with both operands in three bf16 terms (S^T from S staged in
// fp32, rows SROW words apart; G's terms staged in stg[0..2]): the six
// products down to hi x lo and mid x mid, smallest first (the dropped ones
// are below 2^-26 of |S| |G|).  dX is the sum of many products of growing
// states and can be much smaller than |S| |G|, which is why the two-term
// split is not enough here.  One row tile of dX at a time.
__device__ __forceinline__ void st_times_g3(const float* sS, const unsigned char (*stg)[SLICEB], int lane, State& dX)
{
    const int g = lane >> 2, q = lane & 3;
    const int r = lane & 15, cg = lane >> 4;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        uint32_t sh[2][4], sm_[2][4], sl[2][4];
#pragma unroll
        for (int kt = 0; kt < 2; ++kt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int m = 16 * mt + g + 8 * (i & 1), k = 16 * kt + 2 * q + 8 * (i >> 1);
                split_pair3(sS[k * SROW + m], sS[(k + 1) * SROW + m], sh[kt][i], sm_[kt][i], sl[kt][i]);
            }
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t bh[2][4], bm_[2][4], bl[2][4];    // per k-tile: (b0, b1) of column tiles 2 np, 2 np + 1
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) {
                const int off = (16 * kt + r) * ROWB + (8 * (2 * np + cg)) * 2;
                ldsm_x4_trans(bh[kt], stg[0] + off);
                ldsm_x4_trans(bm_[kt], stg[1] + off);
                ldsm_x4_trans(bl[kt], stg[2] + off);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int nt = 2 * np + j;
                float (&acc)[4] = dX[mt][nt];
                mma_bf16_first(acc, sl[0], bh[0][2 * j], bh[0][2 * j + 1]);
                mma_bf16(acc, sl[1], bh[1][2 * j], bh[1][2 * j + 1]);
#pragma unroll
                for (int kt = 0; kt < 2; ++kt) {
                    mma_bf16(acc, sm_[kt], bm_[kt][2 * j], bm_[kt][2 * j + 1]);
                    mma_bf16(acc, sh[kt], bl[kt][2 * j], bl[kt][2 * j + 1]);
                }
#pragma unroll
                for (int kt = 0; kt < 2; ++kt) {
                    mma_bf16(acc, sm_[kt], bh[kt][2 * j], bh[kt][2 * j + 1]);
                    mma_bf16(acc, sh[kt], bm_[kt][2 * j], bm_[kt][2 * j + 1]);
                }
#pragma unroll
                for (int kt = 0; kt < 2; ++kt) mma_bf16(acc, sh[kt], bh[kt][2 * j], bh[kt][2 * j + 1]);
            }
        }
    }
}

// A fragments of Ls^T (A[m][k] = M[k][m] for k > m, else 0) by
// ldmatrix.trans on M, for the tiles kt >= mt (the others are zero).
__device__ __forceinline__ void load_lst_frags(const unsigned char* xs, int lane, uint32_t (&a)[2][2][4])
{
    const int g = lane >> 2, q = lane & 3, d = 2 * q - g;
    const int r = lane & 7, mh = (lane >> 3) & 1, kh = lane >> 4;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            if (kt < mt) continue;
            uint32_t v[4];
            ldsm_x4_trans(v, xs + (16 * kt + 8 * kh + r) * ROWB + (16 * mt + 8 * mh) * 2);
            if (kt == mt) {
                // element (m, k) = (16 mt + g + 8 (i & 1), 16 kt + 2 q + s + 8 (i >> 1)): k - m = off + d + s
                v[0] = tri_mask(v[0], 0, d, true);
                v[1] = 0u;                                     // k - m <= 7 - 8 < 0
                v[3] = tri_mask(v[3], 0, d, true);             // v[2]: k - m >= 8 - 7 > 0, kept
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) a[mt][kt][i] = v[i];
        }
}

// Apply pass: per chunk G from the gradient entering from the right (Gin)
// down to t0, every dL/dx_t, and dL/dS0 from the first chunk.
__global__ void __launch_bounds__(BAWARPS * 32, 4)
k32b_apply(KParams p, const uint16_t* __restrict__ x, const float* __restrict__ S0, const float* __restrict__ S_fwd,
           const float* __restrict__ dS, const float* __restrict__ Gin, float* __restrict__ dx,
           float* __restrict__ dS0)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    BSmem32<true>& sm = reinterpret_cast<BSmem32<true>*>(smem_raw)[warp];
    const int64_t nchains = p.B * p.H * p.K;
    const int64_t first = (int64_t)blockIdx.x * BAWARPS + warp, stride = (int64_t)gridDim.x * BAWARPS;
    const int64_t tok = p.H * NN;
    const int g = lane >> 2, q = lane & 3, d = 2 * q - g;
    const float a = p.ldu_a;
    BFeed32<true> feed;
    feed.chain = first;
    feed.stride = stride;
    feed.nchains = nchains;
    feed.tok = tok;
    feed.set(p);
    feed.issue(sm, 0, lane, p, x, S_fwd, dS);
    int cs = 0;
    for (int64_t chain = first; chain < nchains; chain += stride) {
        const Chain c = chain_at(p, chain);
        const int64_t seq = c.b * p.H + c.h;
        const int64_t base = (c.b * p.L * p.H + c.h) * NN;
        const bool boundary = c.tend < p.L;
        State G;
        if (boundary) load_state(G, Gin + seq_major(p, c) * NN, N, g, q);
        else load_state(G, dS + base + (c.tend - 1) * tok, N, g, q);
        const int64_t hi = boundary ? c.tend : c.tend - 1, lo = c.tbeg;
        for (int64_t tau = hi; tau >= lo; --tau) {
            if (tau >= 1) {                              // dS_{tau-1}, used at the end of this token
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int gi = lane + 32 * i, row = gi >> 3, c4 = gi & 7;
                    cp_async16(sm.ds[0] + row * DROW + 4 * c4, dS + base + (tau - 1) * tok + row * N + 4 * c4);
                }
            }
            cp_async_commit();
            feed.issue(sm, cs ^ 1, lane, p, x, S_fwd, dS);
            cp_async_wait<2>();                          // this token's x and S (the next stage and dS may fly)
            __syncwarp();
            const unsigned char* xs = sm.x[cs];
            stage_dd_b(p, xs, sm.dd[cs], lane);
            const float* Dv = sm.dd[cs][0];
            uint32_t bmt[2][4][2];
            load_mt_frags(xs, lane, bmt);
            float mdt[2][4][4];
            load_mt_d(xs, g, q, mdt);
            if (tau == c.tend) {                       // G_{t1-1} = dS_{t1-1} + Gin X_{t1}^T
                apply_token_f<false, 3>(G, bmt, mdt, Dv, sm.dd[cs][1], a, lane);
                cp_async_wait<1>();                      // dS_{tau-1}
                __syncwarp();
                add_state(G, sm.ds[0], DROW, g, q);
                __syncwarp();
                cs ^= 1;
                continue;
            }
            // ---- dX = S_{tau-1}^T G (S_{-1} = S0 or I) ----
            State dX;
            {
                uint32_t gh[2][2][4], gm[2][2][4], gl[2][2][4];
                state_frags3(G, gh, gm, gl);
                stage_frags3(sm.stg, gh, gm, gl, g, q);
            }
            if (tau == 0 && S0) {                      // S0 into the (unused) S tile of this stage
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int gi = lane + 32 * i, row = gi >> 3, c4 = gi & 7;
                    *reinterpret_cast<float4*>(&sm.s[cs][0] + row * SROW + 4 * c4) =
                        *reinterpret_cast<const float4*>(S0 + seq * NN + row * N + 4 * c4);
                }
            }
            __syncwarp();
            if (tau >= 1 || S0) {
                st_times_g3(&sm.s[cs][0], sm.stg, lane, dX);
            } else {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) dX[mt][nt][i] = G[mt][nt][i];
            }
            __syncwarp();                              // every lane done with the staged G
            // ---- the LDU chain rule ----
            // P1 = dX U^T = dX + a dX Us^T (lower mask on M^T), P2 = L^T dX = dX + a Ls^T dX
            State acc1, acc2;
            {
                uint32_t dh[2][2][4], dl[2][2][4];
                state_frags(dX, dh, dl);
                tri_product<true>(dh, dl, bmt, d, acc1);
                stage_frags(sm.stg, dh, dl, g, q);
            }
            __syncwarp();
            {
                uint32_t bdh[2][4][2], bdl[2][4][2];
                load_m_frags(sm.stg[0], lane, bdh);
                load_m_frags(sm.stg[1], lane, bdl);
                uint32_t als[2][2][4];
                load_lst_frags(xs, lane, als);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        mma_bf16_first(acc2[mt][nt], als[mt][1], bdl[1][nt][0], bdl[1][nt][1]);
                        if (mt == 0) mma_bf16(acc2[mt][nt], als[mt][0], bdl[0][nt][0], bdl[0][nt][1]);
                        if (mt == 0) mma_bf16(acc2[mt][nt], als[mt][0], bdh[0][nt][0], bdh[0][nt][1]);
                        mma_bf16(acc2[mt][nt], als[mt][1], bdh[1][nt][0], bdh[1][nt][1]);
                    }
            }
            float md[2][4][4];
            load_m_d(xs, g, q, md);
            // row sums of (L^T dX)_ik M_ik over k > i, for this lane's rows (mt, h)
            float rs[2][2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float v = 0.0f;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int s2 = 0; s2 < 2; ++s2) {
                            const int i = 2 * h + s2, R = 2 * mt + h, cs2 = 2 * q + s2;
                            const bool above = R < nt || (R == nt && cs2 > g);
                            if (above) v = fmaf(fmaf(a, acc2[mt][nt][i], dX[mt][nt][i]), md[mt][nt][i], v);
                        }
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    rs[mt][h] = v;
                }
            float* out = dx + base + tau * tok;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = 16 * mt + g + 8 * h, R = 2 * mt + h;
                        const float dr = Dv[row];
                        float o[2];
#pragma unroll
                        for (int s2 = 0; s2 < 2; ++s2) {
                            const int i = 2 * h + s2, cs2 = 2 * q + s2, col = 8 * nt + cs2;
                            const float p1 = fmaf(a, acc1[mt][nt][i], dX[mt][nt][i]);
                            const float p2 = fmaf(a, acc2[mt][nt][i], dX[mt][nt][i]);
                            const bool below = R > nt || (R == nt && g > cs2);
                            const bool diag = R == nt && g == cs2;
                            if (below) o[s2] = a * p1 * Dv[col];
                            else if (diag) o[s2] = fmaf(a, rs[mt][h], p2) * dr * sm.dd[cs][2][row];
                            else o[s2] = a * dr * p2;
                        }
                        *reinterpret_cast<float2*>(out + row * N + 8 * nt + 2 * q) = make_float2(o[0], o[1]);
                    }
            // ---- G_{tau-1} = dS_{tau-1} + G X_tau^T, or dS0 = G X_0^T at the first token ----
            if (tau > lo || tau == 0) {
                apply_token_f<false, 3>(G, bmt, mdt, Dv, sm.dd[cs][1], a, lane);
                if (tau == 0) {
                    if (dS0) store_state(dS0 + seq * NN, G, g, q);
                } else {
                    cp_async_wait<1>();                  // dS_{tau-1}
                    __syncwarp();
                    add_state(G, sm.ds[0], DROW, g, q);
                }
            }
            __syncwarp();
            cs ^= 1;
        }
    }
}

// CTAs of a persistent launch: resident CTAs per SM times the SM count,
// cached per device and kernel slot; no more than the chains need.
std::atomic<int> g_resident[64][4];

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

// The same for a kernel with its own block shape (backward kernels).
cudaError_t persistent_grid_w(int slot, const void* kern, int threads, size_t smem, int warps, int64_t nchains,
                              unsigned& grid)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
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

bool supports_backward(const KParams& p)
{
    return p.n == N && p.src == SRC_EMBEDDING && p.x_dtype == MRU_BF16 && p.mode == MRU_MODE_LDU &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_BF16X3) && p.chunk > 0;
}

cudaError_t launch_bwd_local(const KParams& p, const void* x, const float* dS, float* gloc, float* Wq,
                             cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(BSmem32<false>) * BLWARPS;
    cudaError_t e = cudaFuncSetAttribute(k32b_local, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    if ((e = persistent_grid_w(2, (const void*)k32b_local, BLWARPS * 32, sm, BLWARPS, nchains, grid)) != cudaSuccess)
        return e;
    k32b_local<<<grid, BLWARPS * 32, sm, s>>>(p, reinterpret_cast<const uint16_t*>(x), dS, gloc, Wq);
    return cudaGetLastError();
}

cudaError_t launch_bwd_apply(const KParams& p, const void* x, const float* S0, const float* S_fwd, const float* dS,
                             const float* Gin, float* dx, float* dS0, cudaStream_t s)
{
    const int64_t nchains = p.B * p.H * p.K;
    if (nchains == 0) return cudaSuccess;
    if (nchains >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const size_t sm = sizeof(BSmem32<true>) * BAWARPS;
    cudaError_t e = cudaFuncSetAttribute(k32b_apply, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    if ((e = persistent_grid_w(3, (const void*)k32b_apply, BAWARPS * 32, sm, BAWARPS, nchains, grid)) != cudaSuccess)
        return e;
    k32b_apply<<<grid, BAWARPS * 32, sm, s>>>(p, reinterpret_cast<const uint16_t*>(x), S0, S_fwd, dS, Gin, dx, dS0);
    return cudaGetLastError();
}

}  // namespace n32
}  // namespace mru
