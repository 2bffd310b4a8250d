// mru_internal.cuh -- shared device-side definitions of libmru (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mru.h"

namespace mru {

// Source of the per-token matrices a kernel consumes.
enum Source : int32_t {
    SRC_EMBEDDING = 0,   // construct X from the embedding x (mode, alpha, ...)
    SRC_X = 1,           // read X, use F = X - I
    SRC_F = 2            // read F = X - I directly
};

// Bits of the device status word (first 4 bytes of the workspace).
enum : uint32_t { STATUS_SINGULAR = 1u, STATUS_TIMEOUT = 2u };

// Everything a kernel needs to know about the problem, by value.
struct KParams {
    int64_t B, H, L;
    int32_t n;
    int32_t x_dtype;
    int32_t mode;
    int32_t src;
    float alpha;
    int32_t add_identity;
    float ldu_a;
    float ldu_d;
    int32_t math;        // mru_math requested
    int32_t chunk;       // tokens per chunk (C)
    int64_t K;           // chunks per sequence, ceil(L / C)
    int32_t group;       // chunk totals per carry group (G)
    int64_t NG;          // carry groups per sequence, ceil(K / G)
    // q = (umulhi(i, mul) + i) >> shr is i / H (i / K) for 0 <= i < 2^31
    uint32_t h_mul, h_shr, k_mul, k_shr;
    // readout: query columns of U (o_t = S_t U, [n, rq] per token and head)
    // and the distance between heads' U in floats (0: one U for all heads)
    int32_t rq;
    int64_t u_hs;
};

// Multiplier and shift of the division by d (>= 1) for 31-bit dividends:
// l = ceil(log2 d), mul = floor(2^32 (2^l - d) / d) + 1 (Granlund and
// Montgomery, 1994, unsigned division by invariant integers).
inline void fastdiv_magic(int64_t d, uint32_t& mul, uint32_t& shr)
{
    if (d <= 1) { mul = 0; shr = 0; return; }
    uint32_t l = 0;
    while ((int64_t(1) << l) < d) ++l;
    const unsigned __int128 num = ((unsigned __int128)1 << 32) * (((unsigned __int128)1 << l) - (unsigned __int128)d);
    mul = (uint32_t)(num / (unsigned __int128)d + 1);
    shr = l;
}
__device__ __forceinline__ uint32_t fastdiv(uint32_t i, uint32_t mul, uint32_t shr)
{
    return (__umulhi(i, mul) + i) >> shr;
}

// Workspace carve-up (byte offsets from the workspace base).
// Multi-level fp64 scan of chunk totals (mru_carry.cu).
namespace carry {
constexpr int kMaxLevels = 8;
struct Plan {
    int64_t nseq;                 // independent sequences (B * H)
    int G;                        // group size at every level
    int levels;                   // levels below the top
    int64_t cnt[kMaxLevels + 1];  // matrices per sequence at each level
    size_t R[kMaxLevels];         // local prefixes of level l (fp32 for l = 0, else fp64)
    size_t Tot[kMaxLevels];       // group totals of level l (fp64)
    size_t E[kMaxLevels + 1];     // exclusive carries of level l >= 1 (fp64)
    size_t end;                   // first byte after the plan's buffers
};
Plan plan(int64_t nseq, int64_t K, int nn, size_t off);
int launches(const Plan& pl);
cudaError_t run_n32(const Plan& pl, const float* totals, const float* S0, char* ws, cudaStream_t s, int& slot);
}  // namespace carry

// n = 16 carry scan (one launch between the passes): a warp per group of G
// chunk totals scans the group (fp64 tensor cores) and passes the group total
// up a level; the last warp of a group there scans it, up to the top, which
// is scanned from S0.
namespace n16 {
constexpr int kCarryLevels = 3;
struct CarryPlan {
    int64_t nseq;
    int32_t G, gshift;                   // items per group, a power of two (G = 1 << gshift)
    int32_t levels;                      // scanned levels below the top (<= kCarryLevels)
    int64_t cnt[kCarryLevels + 1];       // items per sequence at level l (cnt[0] = K chunk totals)
    size_t R[kCarryLevels];              // inclusive in-group prefixes of level l, [seq][cnt[l]] (fp32 at l = 0, else fp64)
    size_t Tot[kCarryLevels];            // group totals of level l (fp64), [seq][cnt[l + 1]]
    size_t Etop;                         // exclusive carries of the top level (fp64), [seq][cnt[levels]]
    size_t ctr[kCarryLevels + 1];        // arrival counters (uint32): level l [seq][cnt[l + 1]], top [seq]
    size_t ctr_begin, ctr_bytes;         // the counters (zeroed by every reduce launch)
    size_t end;
};
// Workspace of the single-read fused kernel (k16_fused): chunk totals and
// in-group prefixes per chunk, group aggregates, carries and inclusive
// prefixes per group of 2^gshift chunks, per-token scalars of the corrected
// mode, and a control block (tickets, abort flag, group counters and flags)
// that is zeroed before every launch.
struct FusedPlan {
    int32_t gshift;
    int64_t NG, Lp;                      // groups per sequence; row length of the scalar records
    size_t tot, R0, agg, incl, excl, cd;
    size_t ctl, gcnt, gflag, ctl_bytes;  // control block [ctl, ctl + ctl_bytes)
    size_t end;
};
}  // namespace n16

struct Workspace {
    size_t status;       // uint32 status word
    size_t totals;       // float  [B*H, K, n, n]   chunk totals, split form (T - I)
    size_t local;        // double [B*H, K, n, n]   inclusive in-group prefixes of totals, split form
    size_t gcarry;       // double [B*H, NG, n, n]  exclusive group carries (full matrices)
    size_t carry;        // float  [B*H, K, n, n]   exclusive chunk carries (full matrices)
    bool fast;           // specialised kernels: chunk totals and a carry plan
    int fast_n;          // 16 or 32: which specialised kernels
    carry::Plan plan;    // n = 32
    n16::CarryPlan c16;  // n = 16, three launches
    n16::FusedPlan f16;  // n = 16, the single-read fused launch
    bool fused;          // n = 16 runs k16_fused
    size_t fbuf;         // float [B, L, H, n, n]: F = X - I of an orthogonal construction, written by the
    bool fstore;         // reduce pass and read by the apply pass (n = 16, Cayley or exponential)
    size_t bytes;        // total
};

// Backward workspace (mru_scan_backward).
struct BwdWorkspace {
    size_t status;       // uint32 status word
    size_t gloc;         // float [B*H, K, n, n]  local gradient at each chunk's first token
    size_t wq;           // float [B*H, K, n, n]  W_k - I, W_k = X_{t0+1} ... X_{t1}
    size_t gin;          // float [B*H, K, n, n]  gradient entering each chunk from the right
    // The chunk-gradient scan in groups of G = 2^gshift chunks (NG per
    // sequence): per chunk the composition of the maps of the later chunks of
    // its group (g part, W part in split form), per group its whole
    // composition and the gradient entering its last chunk (all fp64).
    int32_t gshift;
    int64_t NG;
    size_t sg, sw;       // double [B*H, K, n, n]
    size_t gg, gw, ginr; // double [B*H, NG, n, n]
    size_t bytes;
};

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Packed fp32 pairs (sm_100): one instruction applies the operation to both
// halves of a 64-bit register pair, each half rounded to nearest as the
// scalar instruction would (results equal the scalar ones bit for bit); the
// FLOP rate is the scalar one, the issue slots halve.
namespace f2 {
__device__ __forceinline__ uint64_t pk(float a, float b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void up(uint64_t r, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
}  // namespace f2

// Workspace bytes mru_scan_fused needs for this problem and output form
// (mru_api.cu); 0 for an invalid problem.
size_t fused_workspace_bytes(const mru_problem& p, const mru_readout* ro);

// Benchmark hook (mru_api.cu): records the caller's event for kernel slot
// `kernel`, before (after = 0) or after (after = 1) its launch; no-op when
// no events are registered.
void profile_mark(int kernel, int after, cudaStream_t s);

// n = 16 tensor-core kernels (mru_n16.cu).
namespace n16 {
constexpr int kSub = 8;           // chunks of the specialised kernels are multiples of it
bool supports(const KParams& p, bool readout);
int32_t preferred_chunk(int64_t token_heads);
CarryPlan carry_plan(int64_t nseq, int64_t K, size_t off);
// fout: for the Cayley map and the exponential, where every token's F = X - I
// goes (x's layout) for the apply pass to read, or null.
cudaError_t launch_reduce(const KParams& p, const float* x, float* totals, const CarryPlan& cp, char* ws,
                          uint32_t* status, float* fout, cudaStream_t s);
cudaError_t launch_carry(const KParams& p, const float* totals, const CarryPlan& cp, char* ws, const float* S0,
                         cudaStream_t s);
// direct: a single-chunk problem (K = 1), run by the apply pass alone with
// the carry S0 (or I when S0 is null); no reduce or carry launch precedes it.
// pre_transformed: x holds the F = X - I the reduce pass wrote (not direct).
cudaError_t launch_apply(const KParams& p, const float* x, const CarryPlan& cp, const char* ws, float* S_out,
                         uint32_t* status, const float* S0, bool direct, bool pre_transformed, cudaStream_t s);
// The single-read fused scan (one launch after a memset of its control block).
FusedPlan fused_plan(const KParams& p, size_t off);
cudaError_t launch_fused(const KParams& p, const FusedPlan& fp, char* ws, const float* x, const float* S0,
                         float* S_out, uint32_t* status, cudaStream_t s);
// Testing hook: the next fused launch never publishes its first group's carry
// and bounds its waits by `ms` milliseconds, so that it ends with
// STATUS_TIMEOUT.
void set_stall_test(int32_t ms);
// Backward passes on the tensor cores (fp32 embeddings, reshape, and the
// determinant-corrected mode with the identity); the generic fp64 scan of
// the chunk gradients runs between them.
bool supports_backward(const KParams& p);
cudaError_t launch_bwd_local(const KParams& p, const float* x, const float* dS, float* gloc, float* Wq,
                             uint32_t* status, cudaStream_t s);
cudaError_t launch_bwd_apply(const KParams& p, const float* x, const float* S0, const float* S_fwd, const float* dS,
                             const float* Gin, float* dx, float* dS0, uint32_t* status, cudaStream_t s);
}  // namespace n16

// n = 32 LDU tensor-core kernels (mru_n32.cu).
namespace n32 {
bool supports(const KParams& p, bool readout);
int32_t preferred_chunk(int64_t token_heads);
cudaError_t launch_reduce(const KParams& p, const void* x, float* totals, cudaStream_t s);
cudaError_t launch_apply(const KParams& p, const void* x, const carry::Plan& pl, const char* ws, float* S_out,
                         const float* S0, bool direct, cudaStream_t s);
// Backward of the LDU scan (bf16 embeddings): local pass and apply pass; the
// chunk-gradient scan between them is the generic one.
bool supports_backward(const KParams& p);
cudaError_t launch_bwd_local(const KParams& p, const void* x, const float* dS, float* gloc, float* Wq,
                             cudaStream_t s);
cudaError_t launch_bwd_apply(const KParams& p, const void* x, const float* S0, const float* S_fwd, const float* dS,
                             const float* Gin, float* dx, float* dS0, cudaStream_t s);
}  // namespace n32

// n = 64 readout chunk kernel on the tensor cores (mru_n64.cu); the carry
// scan and fix-up are the generic kernels.
namespace n64 {
bool supports(const KParams& p, bool readout);
// The chunk phase on tcgen05 (k64_chunk_readout_tc) instead of mma.sync:
// MRU_N64_TCGEN05=1 in the environment, read at every call.
bool use_tcgen05();
cudaError_t launch_chunk_readout(const KParams& p, const float* x, const float* u, int64_t snap_every,
                                 float* o_out, float* snaps, float* totals, uint32_t* status, cudaStream_t s);
// o_t = C U + C V_t and the snapshots C + C Q_t from the chains' carries C.
cudaError_t launch_fixup_readout(const KParams& p, const float* carry, const float* u, int64_t snap_every,
                                 float* o_out, float* snaps, cudaStream_t s);
// Backward on the tensor cores (mru_n64_bwd.cu) when tf32 is asked for:
// local pass and apply pass; the chunk-gradient scan between them is the
// generic one.
bool supports_backward(const KParams& p);
cudaError_t launch_bwd_local(const KParams& p, const float* x, const float* dS, float* gloc, float* Wq,
                             uint32_t* status, cudaStream_t s);
cudaError_t launch_bwd_apply(const KParams& p, const float* x, const float* S0, const float* S_fwd, const float* dS,
                             const float* Gin, float* dx, float* dS0, uint32_t* status, cudaStream_t s);
}  // namespace n64

// Launchers (mru_scan_v1.cu).
cudaError_t launch_build_states(const KParams& p, const void* x, float* X_out, int store_minus_identity,
                                void* ws_base, const Workspace& W, cudaStream_t s);
cudaError_t launch_scan(const KParams& p, const void* src, const float* S0, const float* u,
                        int64_t snap_every, float* S_out, float* o_out, float* snaps,
                        void* ws_base, const Workspace& W, cudaStream_t s, int* launches);
cudaError_t launch_backward(const KParams& p, const void* x, const float* S0, const float* S_fwd, const float* dS,
                            float* dx, float* dS0, void* ws_base, const BwdWorkspace& W, cudaStream_t s);
// dL/dS_t = do_t U^T (+ the snapshot's gradient at 1-based t = k * every)
// for every state, the upstream gradient of the readout form (mru_readout_bwd.cu).
cudaError_t launch_readout_grad(const KParams& p, const float* u, int q, int64_t u_hs, const float* d_o,
                                int64_t every, const float* d_snap, float* dS, cudaStream_t s);
// Name of the i-th kernel one launch_scan call starts for this problem.
const char* kernel_name(const KParams& p, bool readout, int i);
// mru_math the kernels for this problem actually use (MRU_MATH_FP32 for the
// generic kernels).
int32_t effective_math(const KParams& p, bool readout);

}  // namespace mru
