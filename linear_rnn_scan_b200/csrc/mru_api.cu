// mru_api.cu -- the extern "C" boundary of libmru: argument checks, workspace
// layout, kernel selection and launch.  No allocation happens here: every
// buffer, the workspace included, belongs to the caller.
#include <stdlib.h>
#include <string.h>

#include "mru_internal.cuh"

namespace mru {
namespace {

bool supported_n(int n) { return n == 4 || n == 8 || n == 16 || n == 32 || n == 64; }

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Tokens per chunk of the generic path: aim at about 4096 chains (b, h,
// chunk) so that a launch fills 148 SMs several times over; a power of two
// in [16, 1024].
int32_t generic_chunk(const mru_problem& p)
{
    const int64_t th = p.B * p.H * p.L;
    int64_t c = 16;
    while (c < 1024 && c * 4096 < th) c *= 2;
    return (int32_t)c;
}

// Whether the fused scan of this problem (with or without the readout) runs
// on the specialised n = 16 kernels, given the chunk they need.
bool fast16_eligible(const mru_problem& p, bool readout)
{
    return p.n == 16 && p.x_dtype == MRU_F32 && !readout &&
           (p.mode == MRU_MODE_RESHAPE || p.mode == MRU_MODE_DETNORM || p.mode == MRU_MODE_CAYLEY ||
            p.mode == MRU_MODE_EXPM) &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_TF32X3) && p.chunk % n16::kSub == 0;
}

bool fast32_eligible(const mru_problem& p, bool readout)
{
    return p.n == 32 && p.x_dtype == MRU_BF16 && !readout && p.mode == MRU_MODE_LDU &&
           (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_BF16X3) && p.chunk % n16::kSub == 0;
}

// The n = 64 readout path (one CTA per chain): the longest chunk up to 128
// tokens that still leaves 1,024 chains (about 1.7 waves of resident CTAs);
// longer chunks mean fewer chunk totals for the carry scan and the fix-up.
// Measured on B200 for B2 H4 L16384: 32 -> 2.56 ms, 64 -> 2.25, 128 -> 2.15,
// 256 -> 2.34.
// Every state (no readout) takes the same path when tf32 is asked for
// explicitly (the fix-up writes each token's state as a snapshot).
bool fast64_eligible(const mru_problem& p, bool readout)
{
    return p.n == 64 && p.x_dtype == MRU_F32 && (p.mode == MRU_MODE_DETNORM || p.mode == MRU_MODE_RESHAPE) &&
           (readout ? (p.math == MRU_MATH_AUTO || p.math == MRU_MATH_TF32) : p.math == MRU_MATH_TF32);
}

int32_t n64_chunk(int64_t token_heads)
{
    int32_t c = 16;
    while (c < 128 && token_heads / (2 * (int64_t)c) >= 1024) c *= 2;
    return c;
}

// n = 4 without a readout, sequences of up to 16384 tokens, and either at
// most 2^20 tokens in all or at least one sequence per SM: the whole
// sequence is one chunk, run by the one-launch kernel (one CTA per
// sequence, up to 64 tokens per thread; 18x faster than the passes at
// 1024 sequences of 1024 tokens).  Few long sequences keep the passes.
bool small_eligible(const mru_problem& p, int32_t src, bool readout)
{
    return p.n == 4 && !readout && p.L >= 1 && p.L <= 16384 && p.B * p.H < (int64_t(1) << 31) &&
           (p.B * p.H * p.L <= (int64_t(1) << 20) || p.B * p.H >= 148) &&
           (src != SRC_EMBEDDING || p.mode == MRU_MODE_RESHAPE || p.mode == MRU_MODE_DETNORM ||
            p.mode == MRU_MODE_LDU);
}

int32_t choose_chunk(const mru_problem& p, int32_t src, bool readout)
{
    if (p.chunk > 0) return p.chunk;
    if (small_eligible(p, src, readout)) return (int32_t)p.L;
    if (src == SRC_EMBEDDING && fast64_eligible(p, readout)) return n64_chunk(p.B * p.H * p.L);
    if (src == SRC_EMBEDDING && fast32_eligible(p, readout)) return n32::preferred_chunk(p.B * p.H * p.L);
    if (src == SRC_EMBEDDING && fast16_eligible(p, readout))
        return n16::preferred_chunk(p.B * p.H * p.L);
    return generic_chunk(p);
}

int32_t choose_group(int64_t K)
{
    int64_t g = 1;
    while (g * g < K) ++g;
    return (int32_t)(g < 1 ? 1 : g);
}

mru_status check_problem(const mru_problem* p)
{
    if (!p) return MRU_ERR_INVALID_ARG;
    if (p->B < 0 || p->H < 0 || p->L < 0 || p->chunk < 0) return MRU_ERR_INVALID_ARG;
    if (p->x_dtype != MRU_F32 && p->x_dtype != MRU_BF16) return MRU_ERR_INVALID_ARG;
    if (p->mode < MRU_MODE_RESHAPE || p->mode > MRU_MODE_EXPM) return MRU_ERR_INVALID_ARG;
    if (p->math < MRU_MATH_AUTO || p->math > MRU_MATH_BF16X3) return MRU_ERR_INVALID_ARG;
    if (p->add_identity != 0 && p->add_identity != 1) return MRU_ERR_INVALID_ARG;
    if (!supported_n(p->n)) return MRU_ERR_UNSUPPORTED;
    return MRU_OK;
}

KParams make_params(const mru_problem& p, int32_t src, bool readout)
{
    KParams k;
    memset(&k, 0, sizeof k);
    k.B = p.B; k.H = p.H; k.L = p.L; k.n = p.n;
    k.x_dtype = p.x_dtype; k.mode = p.mode; k.src = src;
    k.alpha = p.alpha; k.add_identity = p.add_identity;
    k.ldu_a = p.ldu_offdiag; k.ldu_d = p.ldu_diag;
    k.math = p.math;
    k.chunk = choose_chunk(p, src, readout);
    k.K = ceil_div(p.L, k.chunk);
    k.group = choose_group(k.K);
    k.NG = k.K > 0 ? ceil_div(k.K, k.group) : 0;
    fastdiv_magic(k.H, k.h_mul, k.h_shr);
    fastdiv_magic(k.K, k.k_mul, k.k_shr);
    k.rq = 1;
    return k;
}

// The single-read fused n = 16 kernel is opt-in (MRU_N16_FUSED=1 in the
// environment, read at each call): on B200 it is still slower than the three
// passes (configuration B8 H8 L4096: 0.34 ms against 0.22 ms), its warps
// waiting on group carries.
bool fused16_enabled()
{
    const char* v = getenv("MRU_N16_FUSED");
    return v && v[0] == '1';
}

// fstore_ok: the n = 16 passes of the Cayley map and the exponential may keep
// every token's F = X - I in the workspace (written by the reduce pass, read
// by the apply pass instead of forming F again); off, they form it twice.
Workspace layout(const KParams& k, bool readout, bool fstore_ok = true)
{
    Workspace W;
    memset(&W, 0, sizeof W);
    const size_t nn = (size_t)k.n * k.n;
    const size_t BH = (size_t)(k.B * k.H);
    size_t off = 0;
    W.status = off; off += 256;
    if (n16::supports(k, readout)) {
        W.fast = true;
        W.fast_n = 16;
        W.fused = fused16_enabled();
        if (W.fused) {
            W.f16 = n16::fused_plan(k, off);
            W.bytes = W.f16.end;
            return W;
        }
        W.totals = off; off = round_up(off + BH * k.K * nn * sizeof(float), 256);
        W.c16 = n16::carry_plan((int64_t)BH, k.K, off);
        off = W.c16.end > off ? W.c16.end : off;
        if (fstore_ok && k.K > 1 && (k.mode == MRU_MODE_CAYLEY || k.mode == MRU_MODE_EXPM)) {
            W.fstore = true;
            W.fbuf = off;
            off = round_up(off + (size_t)k.B * (size_t)k.L * (size_t)k.H * nn * sizeof(float), 256);
        }
        W.bytes = off;
        return W;
    }
    if (n32::supports(k, readout)) {
        W.fast = true;
        W.fast_n = 32;
        W.totals = off; off = round_up(off + BH * k.K * nn * sizeof(float), 256);
        W.plan = carry::plan((int64_t)BH, k.K, (int)nn, off);
        W.bytes = W.plan.end > off ? W.plan.end : off;
        return W;
    }
    W.totals = off; off = round_up(off + BH * k.K * nn * sizeof(float), 256);
    W.local = off;  off = round_up(off + BH * k.K * nn * sizeof(double), 256);
    W.gcarry = off; off = round_up(off + BH * k.NG * nn * sizeof(double), 256);
    W.carry = off;  off = round_up(off + BH * k.K * nn * sizeof(float), 256);
    W.bytes = off;
    return W;
}

// The backward's chunking: the generic chunk (or the caller's) and its
// workspace.
// The n = 64 tensor-core backward: chunks of 64 tokens while that leaves
// 1,184 chains (four waves of two CTAs per SM on 148 SMs; measured on B200
// for B2 H4 L16384: 6.14 ms with chunks of 64, 6.38 with 32, 6.55 with 128),
// halved down to 8 for smaller problems.
int32_t n64_bwd_chunk(const mru_problem& p)
{
    const int64_t th = p.B * p.H * p.L;
    int64_t c = 64;
    while (c > 8 && th / c < 1184) c /= 2;
    return (int32_t)c;
}

KParams make_bwd_params(const mru_problem& p)
{
    KParams k = make_params(p, SRC_EMBEDDING, false);
    k.chunk = p.chunk > 0 ? p.chunk : (n64::supports_backward(k) ? n64_bwd_chunk(p) : generic_chunk(p));
    k.K = ceil_div(p.L, k.chunk);
    fastdiv_magic(k.K, k.k_mul, k.k_shr);
    return k;
}

BwdWorkspace bwd_layout(const KParams& k)
{
    BwdWorkspace W;
    memset(&W, 0, sizeof W);
    const size_t nn = (size_t)k.n * k.n, chains = (size_t)(k.B * k.H * k.K);
    size_t off = 0;
    W.status = off; off += 256;
    W.gloc = off; off = round_up(off + chains * nn * sizeof(float), 256);
    W.wq = off;   off = round_up(off + chains * nn * sizeof(float), 256);
    W.gin = off;  off = round_up(off + chains * nn * sizeof(float), 256);
    // groups of about sqrt(K) chunks: the serial steps are G within the groups
    // and NG across them
    W.gshift = 0;
    while (((int64_t)1 << (2 * W.gshift)) < k.K) ++W.gshift;
    W.NG = k.K > 0 ? (k.K + ((int64_t)1 << W.gshift) - 1) >> W.gshift : 0;
    const size_t groups = (size_t)(k.B * k.H) * (size_t)W.NG;
    W.sg = off;   off = round_up(off + chains * nn * sizeof(double), 256);
    W.sw = off;   off = round_up(off + chains * nn * sizeof(double), 256);
    W.gg = off;   off = round_up(off + groups * nn * sizeof(double), 256);
    W.gw = off;   off = round_up(off + groups * nn * sizeof(double), 256);
    W.ginr = off; off = round_up(off + groups * nn * sizeof(double), 256);
    W.bytes = off;
    return W;
}

cudaEvent_t g_prof_events[64];
int g_prof_count = 0;

mru_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MRU_OK : MRU_ERR_CUDA; }

mru_status reset_status(void* ws, cudaStream_t s)
{
    return from_cuda(cudaMemsetAsync(ws, 0, sizeof(uint32_t), s));
}

}  // namespace

namespace {
// Kernel parameters and workspace layout of one mru_scan_fused call: the
// embedding source, and the readout's query columns when there is one.  The
// layout that keeps F in the workspace is taken when ws_bytes holds it, else
// the one that forms F twice.
void fused_call_plan(const mru_problem& p, const mru_readout* ro, KParams& k, Workspace& W, size_t ws_bytes)
{
    k = make_params(p, SRC_EMBEDDING, ro != nullptr);
    if (ro) {
        k.rq = ro->q == 0 ? 1 : ro->q;
        k.u_hs = ro->u_per_head ? (int64_t)p.n * k.rq : 0;
    }
    W = layout(k, ro != nullptr, true);
    if (W.bytes > ws_bytes) W = layout(k, ro != nullptr, false);
}
}  // namespace

// The least workspace mru_scan_fused accepts for this problem with this
// output form (the readout's query-column count and per-head layout
// included); 0 for an invalid problem.
size_t fused_workspace_bytes(const mru_problem& p, const mru_readout* ro)
{
    if (check_problem(&p) != MRU_OK) return 0;
    KParams k;
    Workspace W;
    fused_call_plan(p, ro, k, W, 0);
    return W.bytes;
}

void profile_mark(int kernel, int after, cudaStream_t s)
{
    const int slot = 2 * kernel + after;
    if (slot < g_prof_count) cudaEventRecord(g_prof_events[slot], s);
}

}  // namespace mru

using namespace mru;

extern "C" {

size_t mru_workspace_size(const mru_problem* p)
{
    if (check_problem(p) != MRU_OK) return 0;
    // large enough for every entry point and for both output forms
    size_t b = 0;
    for (int32_t src : {SRC_EMBEDDING, SRC_X})
        for (bool ro : {false, true}) {
            const size_t w = layout(make_params(*p, src, ro), ro).bytes;
            if (w > b) b = w;
        }
    return b;
}

int32_t mru_effective_math(const mru_problem* p, int32_t readout)
{
    if (check_problem(p) != MRU_OK) return -1;
    const KParams k = make_params(*p, SRC_EMBEDDING, readout != 0);
    return effective_math(k, readout != 0);
}

int32_t mru_chosen_chunk(const mru_problem* p, int32_t readout)
{
    if (check_problem(p) != MRU_OK) return 0;
    return choose_chunk(*p, SRC_EMBEDDING, readout != 0);
}

const char* mru_kernel_name(const mru_problem* p, int32_t readout, int32_t i)
{
    if (check_problem(p) != MRU_OK) return "";
    const KParams k = make_params(*p, SRC_EMBEDDING, readout != 0);
    const Workspace W = layout(k, readout != 0);
    if (!W.fast) return kernel_name(k, readout != 0, i);
    if (k.K == 1) return i == 0 ? (W.fast_n == 16 ? "k16_apply" : "k32_apply") : "";
    if (W.fast_n == 16 && W.fused) return i == 0 ? "k16_fused" : "";
    if (W.fast_n == 16) return i == 0 ? "k16_reduce" : i == 1 ? "k16_carry" : i == 2 ? "k16_apply" : "";
    const int lv = W.plan.levels;
    const bool n32k = W.fast_n == 32;
    if (i == 0) return n32k ? "k32_reduce" : "k16_reduce";
    if (i >= 1 && i <= lv) return "k_level";
    if (i == lv + 1) return "k_top";
    if (i >= lv + 2 && i <= 2 * lv) return "k_down";
    if (i == 2 * lv + 1) return n32k ? "k32_apply" : "k16_apply";
    return "";
}

int32_t mru_launch_count(const mru_problem* p, int32_t readout)
{
    if (check_problem(p) != MRU_OK) return 0;
    if (p->B * p->H * p->L == 0) return 0;
    const KParams k = make_params(*p, SRC_EMBEDDING, readout != 0);
    const Workspace W = layout(k, readout != 0);
    if (k.K == 1) return 1;                  // single chunk: one kernel, from S0
    if (W.fast) return W.fast_n == 16 ? (W.fused ? 1 : 3) : 2 + carry::launches(W.plan);
    return 5;
}

mru_status mru_build_states(const mru_problem* p, const void* x, float* X_out, void* ws, size_t ws_bytes,
                            void* stream)
{
    mru_status st = check_problem(p);
    if (st != MRU_OK) return st;
    if (!x || !X_out || !ws || !aligned16(x) || !aligned16(X_out) || !aligned16(ws)) return MRU_ERR_INVALID_ARG;
    KParams k = make_params(*p, SRC_EMBEDDING, false);
    Workspace W = layout(k, false);
    if (ws_bytes < W.bytes) return MRU_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = reset_status(ws, s)) != MRU_OK) return st;
    if (p->B * p->H * p->L == 0) return MRU_OK;
    return from_cuda(launch_build_states(k, x, X_out, p->store_minus_identity, ws, W, s));
}

mru_status mru_scan(const mru_problem* p, const float* X, const float* S0, float* S_out, void* ws,
                    size_t ws_bytes, void* stream)
{
    mru_status st = check_problem(p);
    if (st != MRU_OK) return st;
    if (!X || !S_out || !ws || !aligned16(X) || !aligned16(S_out) || !aligned16(ws)) return MRU_ERR_INVALID_ARG;
    if (S0 && !aligned16(S0)) return MRU_ERR_INVALID_ARG;
    if ((const void*)X == (const void*)S_out) return MRU_ERR_INVALID_ARG;
    KParams k = make_params(*p, p->store_minus_identity ? SRC_F : SRC_X, false);
    Workspace W = layout(k, false);
    if (ws_bytes < W.bytes) return MRU_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = reset_status(ws, s)) != MRU_OK) return st;
    if (p->B * p->H * p->L == 0) return MRU_OK;
    return from_cuda(launch_scan(k, X, S0, nullptr, 0, S_out, nullptr, nullptr, ws, W, s, nullptr));
}

mru_status mru_scan_fused(const mru_problem* p, const void* x, const float* S0, const mru_readout* ro,
                          float* S_out, float* o_out, void* ws, size_t ws_bytes, void* stream)
{
    mru_status st = check_problem(p);
    if (st != MRU_OK) return st;
    if (!x || !ws || !aligned16(x) || !aligned16(ws)) return MRU_ERR_INVALID_ARG;
    if (S0 && !aligned16(S0)) return MRU_ERR_INVALID_ARG;
    int64_t every = 0;
    float* snaps = nullptr;
    if (ro) {
        if (!ro->u || !o_out || !aligned16(o_out) || ro->snapshot_every < 0) return MRU_ERR_INVALID_ARG;
        if (ro->q < 0 || ro->q > p->n || (ro->u_per_head != 0 && ro->u_per_head != 1)) return MRU_ERR_INVALID_ARG;
        every = ro->snapshot_every;
        if (every > 0) {
            snaps = ro->snapshots;
            if (!snaps || !aligned16(snaps)) return MRU_ERR_INVALID_ARG;
        }
        if ((const void*)o_out == x) return MRU_ERR_INVALID_ARG;
    } else {
        if (!S_out || !aligned16(S_out) || (const void*)S_out == x) return MRU_ERR_INVALID_ARG;
    }
    KParams k;
    Workspace W;
    fused_call_plan(*p, ro, k, W, ws_bytes);
    if (ws_bytes < W.bytes) return MRU_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = reset_status(ws, s)) != MRU_OK) return st;
    if (p->B * p->H * p->L == 0) return MRU_OK;
    return from_cuda(launch_scan(k, x, S0, ro ? ro->u : nullptr, every, ro ? nullptr : S_out,
                                 ro ? o_out : nullptr, snaps, ws, W, s, nullptr));
}

mru_status mru_scan_fused_host(const mru_problem* p, const void* x_host, const float* S0, const mru_readout* ro,
                               float* out_host, float* snaps_host, void* x_dev, float* out_dev, void* ws,
                               size_t ws_bytes, int32_t pieces, void* compute_stream, void* h2d_stream,
                               void* d2h_stream)
{
    mru_status st = check_problem(p);
    if (st != MRU_OK) return st;
    if (!x_host || !out_host || !x_dev || !out_dev || !ws || pieces < 0) return MRU_ERR_INVALID_ARG;
    if (!aligned16(x_dev) || !aligned16(out_dev) || !aligned16(ws) || (S0 && !aligned16(S0)))
        return MRU_ERR_INVALID_ARG;
    if ((const void*)out_dev == x_dev) return MRU_ERR_INVALID_ARG;
    int64_t every = 0;
    if (ro) {
        if (!ro->u || ro->snapshot_every < 0) return MRU_ERR_INVALID_ARG;
        if (ro->q < 0 || ro->q > p->n || (ro->u_per_head != 0 && ro->u_per_head != 1)) return MRU_ERR_INVALID_ARG;
        every = ro->snapshot_every;
        if (every > 0 && (!ro->snapshots || !aligned16(ro->snapshots) || !snaps_host)) return MRU_ERR_INVALID_ARG;
    }
    const bool readout = ro != nullptr;
    KParams k = make_params(*p, SRC_EMBEDDING, readout);
    if (ro) {
        k.rq = ro->q == 0 ? 1 : ro->q;
        k.u_hs = ro->u_per_head ? (int64_t)p->n * k.rq : 0;
    }
    Workspace W = layout(k, readout, true);
    if (ws_bytes < W.bytes) W = layout(k, readout, false);
    if (ws_bytes < W.bytes) return MRU_ERR_WORKSPACE;
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(compute_stream);
    cudaStream_t si = reinterpret_cast<cudaStream_t>(h2d_stream);
    cudaStream_t so = reinterpret_cast<cudaStream_t>(d2h_stream);
    if ((st = reset_status(ws, sc)) != MRU_OK) return st;
    if (p->B * p->H * p->L == 0) return MRU_OK;

    // Pieces: along the batch when there are several sequences per head,
    // else along the sequence (each piece started from the previous piece's
    // last state), never finer than one chunk; one piece with the readout
    // of a single batch (its states are not kept).
    const bool along_b = p->B >= 2;
    int64_t np = pieces == 0 ? 8 : pieces;
    if (along_b) np = np < p->B ? np : p->B;
    else if (readout) np = 1;
    else np = np < k.K ? np : k.K;
    if (np > 64) np = 64;
    if (np < 1) np = 1;

    const int64_t nn = (int64_t)p->n * p->n;
    const size_t xb = p->x_dtype == MRU_BF16 ? 2 : 4;
    const int64_t out_tok = readout ? p->H * p->n * k.rq : p->H * nn;   // floats per (b, t)
    const int64_t ls = every > 0 ? p->L / every : 0;
    cudaEvent_t ev[2 * 64 + 2];
    int nev = 0;
    for (int i = 0; i < 2 * np + 2; ++i) {
        if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) break;
        ++nev;
    }
    cudaError_t e = nev == 2 * np + 2 ? cudaSuccess : cudaErrorMemoryAllocation;
    // the copies start after the work already queued on the compute stream
    if (e == cudaSuccess) e = cudaEventRecord(ev[0], sc);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(si, ev[0], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(so, ev[0], 0);
    const char* xh = reinterpret_cast<const char*>(x_host);
    char* xd = reinterpret_cast<char*>(x_dev);
    for (int64_t i = 0; i < np && e == cudaSuccess; ++i) {
        mru_problem sub = *p;
        sub.chunk = k.chunk;                  // the whole problem's chunk: the workspace fits every piece
        int64_t xoff, ooff, soff = 0, nx, no, ns = 0;
        const float* s0 = S0;
        if (along_b) {
            const int64_t b0 = p->B * i / np, b1 = p->B * (i + 1) / np;
            sub.B = b1 - b0;
            xoff = b0 * p->L * p->H * nn;
            nx = sub.B * p->L * p->H * nn;
            ooff = b0 * p->L * out_tok;
            no = sub.B * p->L * out_tok;
            soff = b0 * ls * p->H * nn;
            ns = sub.B * ls * p->H * nn;
            if (S0) s0 = S0 + b0 * p->H * nn;
        } else {
            const int64_t c0 = k.K * i / np, c1 = k.K * (i + 1) / np;    // whole chunks per piece
            const int64_t t0 = c0 * k.chunk, t1 = c1 * k.chunk < p->L ? c1 * k.chunk : p->L;
            sub.L = t1 - t0;
            xoff = t0 * p->H * nn;
            nx = sub.L * p->H * nn;
            ooff = t0 * out_tok;
            no = sub.L * out_tok;
            if (i > 0) s0 = out_dev + (t0 - 1) * out_tok;               // the previous piece's last state
        }
        if ((e = cudaMemcpyAsync(xd + xoff * xb, xh + xoff * xb, (size_t)nx * xb, cudaMemcpyHostToDevice, si)) !=
            cudaSuccess)
            break;
        if ((e = cudaEventRecord(ev[1 + 2 * i], si)) != cudaSuccess) break;
        if ((e = cudaStreamWaitEvent(sc, ev[1 + 2 * i], 0)) != cudaSuccess) break;
        KParams ki = make_params(sub, SRC_EMBEDDING, readout);
        ki.rq = k.rq;
        ki.u_hs = k.u_hs;
        const Workspace Wi = layout(ki, readout, W.fstore);
        e = launch_scan(ki, xd + xoff * xb, s0, ro ? ro->u : nullptr, every, readout ? nullptr : out_dev + ooff,
                        readout ? out_dev + ooff : nullptr, every > 0 ? ro->snapshots + soff : nullptr, ws, Wi, sc,
                        nullptr);
        if (e != cudaSuccess) break;
        if ((e = cudaEventRecord(ev[2 + 2 * i], sc)) != cudaSuccess) break;
        if ((e = cudaStreamWaitEvent(so, ev[2 + 2 * i], 0)) != cudaSuccess) break;
        if ((e = cudaMemcpyAsync(out_host + ooff, out_dev + ooff, (size_t)no * sizeof(float), cudaMemcpyDeviceToHost,
                                 so)) != cudaSuccess)
            break;
        if (ns > 0 && (e = cudaMemcpyAsync(snaps_host + soff, ro->snapshots + soff, (size_t)ns * sizeof(float),
                                           cudaMemcpyDeviceToHost, so)) != cudaSuccess)
            break;
    }
    // the call is complete once the compute stream passes this point
    if (e == cudaSuccess) e = cudaEventRecord(ev[2 * np + 1], so);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sc, ev[2 * np + 1], 0);
    for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);     // released once they complete
    return from_cuda(e);
}

mru_status mru_last_device_status(const void* ws, void* stream)
{
    if (!ws) return MRU_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MRU_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, ws, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) return MRU_ERR_CUDA;
    if (word & STATUS_TIMEOUT) return MRU_ERR_TIMEOUT;
    if (word & STATUS_SINGULAR) return MRU_ERR_SINGULAR;
    return MRU_OK;
}

void mru_debug_stall_next_fused(int32_t ms) { n16::set_stall_test(ms > 0 ? ms : 0); }

mru_status mru_set_profile_events(void* const* events, int32_t count)
{
    if (count < 0 || count > 64 || (count > 0 && !events)) return MRU_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i)
        if (!events[i]) return MRU_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) g_prof_events[i] = reinterpret_cast<cudaEvent_t>(events[i]);
    g_prof_count = count;
    return MRU_OK;
}

const char* mru_status_string(mru_status s)
{
    switch (s) {
        case MRU_OK: return "ok";
        case MRU_ERR_INVALID_ARG: return "invalid argument";
        case MRU_ERR_UNSUPPORTED: return "unsupported problem (n must be 4, 8, 16, 32 or 64)";
        case MRU_ERR_WORKSPACE: return "workspace too small";
        case MRU_ERR_CUDA: return "CUDA error";
        case MRU_ERR_SINGULAR: return "singular input matrix (det = 0 or not finite)";
        case MRU_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

namespace {
// The readout backward's workspace: one region shared by the forward
// recomputation and the backward (the status word at its start, where
// mru_last_device_status reads it), then the recomputed states and their
// upstream gradients (each [B, L, H, n, n] fp32).
struct ReadoutBwdLayout {
    size_t S, dS, region, region_bytes, bytes;
};
ReadoutBwdLayout readout_bwd_layout(const mru_problem& p)
{
    ReadoutBwdLayout R;
    const size_t states = (size_t)(p.B * p.L * p.H) * (size_t)p.n * p.n * sizeof(float);
    const size_t fwd = layout(make_params(p, SRC_EMBEDDING, false), false).bytes;
    const size_t bwd = bwd_layout(make_bwd_params(p)).bytes;
    R.region = 0;
    R.region_bytes = fwd > bwd ? fwd : bwd;
    R.S = round_up(R.region_bytes, 256);
    R.dS = R.S + round_up(states, 256);
    R.bytes = R.dS + round_up(states, 256);
    return R;
}
}  // namespace

size_t mru_backward_readout_workspace_size(const mru_problem* p)
{
    if (check_problem(p) != MRU_OK) return 0;
    return readout_bwd_layout(*p).bytes;
}

mru_status mru_scan_backward_readout(const mru_problem* p, const void* x, const float* S0, const mru_readout* ro,
                                     const float* d_o, const float* d_snaps, float* dx, float* dS0, void* ws,
                                     size_t ws_bytes, void* stream)
{
    mru_status st = check_problem(p);
    if (st != MRU_OK) return st;
    if (!x || !ro || !ro->u || !d_o || !dx || !ws) return MRU_ERR_INVALID_ARG;
    if (ro->q < 0 || ro->q > p->n || (ro->u_per_head != 0 && ro->u_per_head != 1) || ro->snapshot_every < 0)
        return MRU_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dx) || !aligned16(ws) || !aligned16(d_o) || (S0 && !aligned16(S0)) ||
        (dS0 && !aligned16(dS0)) || (d_snaps && !aligned16(d_snaps)))
        return MRU_ERR_INVALID_ARG;
    if ((const void*)dx == x || (const void*)dx == (const void*)d_o) return MRU_ERR_INVALID_ARG;
    if (dS0 && ((const void*)dS0 == (const void*)S0 || (const void*)dS0 == (const void*)dx)) return MRU_ERR_INVALID_ARG;
    const ReadoutBwdLayout R = readout_bwd_layout(*p);
    if (ws_bytes < R.bytes) return MRU_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* base = reinterpret_cast<char*>(ws);
    char* region = base + R.region;
    if ((st = reset_status(region, s)) != MRU_OK) return st;
    if (p->B * p->H * p->L == 0) {
        if (dS0 && p->B * p->H > 0)
            return from_cuda(cudaMemsetAsync(dS0, 0, sizeof(float) * (size_t)(p->B * p->H * p->n * p->n), s));
        return MRU_OK;
    }
    float* S_buf = reinterpret_cast<float*>(base + R.S);
    float* dS_buf = reinterpret_cast<float*>(base + R.dS);
    cudaError_t e;
    // 1. the states, recomputed by the fused forward (all of them, into the workspace)
    const KParams kf = make_params(*p, SRC_EMBEDDING, false);
    const Workspace Wf = layout(kf, false);
    if ((e = launch_scan(kf, x, S0, nullptr, 0, S_buf, nullptr, nullptr, region, Wf, s, nullptr)) != cudaSuccess)
        return MRU_ERR_CUDA;
    // 2. their upstream gradients from the readout's
    const int q = ro->q == 0 ? 1 : ro->q;
    const int64_t u_hs = ro->u_per_head ? (int64_t)p->n * q : 0;
    if ((e = launch_readout_grad(kf, ro->u, q, u_hs, d_o, ro->snapshot_every, ro->snapshot_every > 0 ? d_snaps : nullptr,
                                 dS_buf, s)) != cudaSuccess)
        return MRU_ERR_CUDA;
    // 3. the scan's backward
    const KParams kb = make_bwd_params(*p);
    const BwdWorkspace Wb = bwd_layout(kb);
    return from_cuda(launch_backward(kb, x, S0, S_buf, dS_buf, dx, dS0, region, Wb, s));
}

size_t mru_backward_workspace_size(const mru_problem* p)
{
    if (check_problem(p) != MRU_OK) return 0;
    return bwd_layout(make_bwd_params(*p)).bytes;
}

mru_status mru_scan_backward(const mru_problem* p, const void* x, const float* S0, const float* S_fwd,
                             const float* dS, float* dx, float* dS0, void* ws, size_t ws_bytes, void* stream)
{
    mru_status st = check_problem(p);
    if (st != MRU_OK) return st;
    if (!x || !S_fwd || !dS || !dx || !ws) return MRU_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(S_fwd) || !aligned16(dS) || !aligned16(dx) || !aligned16(ws))
        return MRU_ERR_INVALID_ARG;
    if ((S0 && !aligned16(S0)) || (dS0 && !aligned16(dS0))) return MRU_ERR_INVALID_ARG;
    if ((const void*)dx == x || (const void*)dx == (const void*)S_fwd || (const void*)dx == (const void*)dS)
        return MRU_ERR_INVALID_ARG;
    if (dS0 && ((const void*)dS0 == (const void*)S0 || (const void*)dS0 == (const void*)dx)) return MRU_ERR_INVALID_ARG;
    const KParams k = make_bwd_params(*p);
    const BwdWorkspace W = bwd_layout(k);
    if (ws_bytes < W.bytes) return MRU_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = reset_status(ws, s)) != MRU_OK) return st;
    if (p->B * p->H * p->L == 0) {
        // no state depends on S0 when L = 0
        if (dS0 && p->B * p->H > 0)
            return from_cuda(cudaMemsetAsync(dS0, 0, sizeof(float) * (size_t)(p->B * p->H * p->n * p->n), s));
        return MRU_OK;
    }
    return from_cuda(launch_backward(k, x, S0, S_fwd, dS, dx, dS0, ws, W, s));
}

}  // extern "C"
