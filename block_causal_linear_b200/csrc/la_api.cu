// la_api.cu -- the C ABI of libla_b200.so (declared in include/la.h).
//
// Host side only: argument validation, the launch plan (split counts), the
// workspace layout, RoPE frequency tables, and the sequence of kernel
// launches of one call.  Every step of the computation runs in the kernels of
// k_ffma.cu, k_finish.cu and k_tc.cu.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/la.h"
#include "la_internal.cuh"

namespace {

int g_last_launches = 0;
const char *g_last_path = "none";
cudaEvent_t g_ev[4] = {nullptr, nullptr, nullptr, nullptr};

// Record stage event i on s.  Under stream capture the record becomes an
// event-record node of the graph (external), so that each replay records it.
inline bool mark(int i, cudaStream_t s) {
    if (!g_ev[i]) return true;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return false;
    const unsigned flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    return cudaEventRecordWithFlags(g_ev[i], s, flags) == cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

// Deterministic split plan: a function of the shapes only (never of the GPU),
// so that results are reproducible bit for bit.  Each block is cut into P
// reduce splits (16-token granularity) and Pa apply splits (128-token tiles)
// so that one wave of at most kTargetCtas CTAs covers the call.
void make_splits(la::Plan &p) {
    const long long groups = (long long)p.B * ceil_div(p.H, 4) * p.nb;
    long long want = la::kTargetCtas / groups;
    if (want > ceil_div(p.L, la::kReduceRows)) want = ceil_div(p.L, la::kReduceRows);
    if (want < 1) want = 1;
    const long long chunk = ceil_div(ceil_div(p.L, want), 16) * 16;
    p.chunk = (int)chunk;
    p.P = (int)ceil_div(p.L, chunk);

    const long long pairs = (long long)p.B * ceil_div(p.H, 2) * p.nb;
    long long wanta = la::kTargetCtas / pairs;
    if (wanta > ceil_div(p.L, la::kApplyRows)) wanta = ceil_div(p.L, la::kApplyRows);
    if (wanta < 1) wanta = 1;
    const long long chunka = ceil_div(ceil_div(p.L, wanta), la::kApplyRows) * la::kApplyRows;
    p.chunka = (int)chunka;
    p.Pa = (int)ceil_div(p.L, chunka);
    // the stream-K plans of the RoPE kernels (the workspace holds their split sums too)
    la::plan_rope_sk(p);
}

// The fused plan (the reduce combines its own splits): one block per call and
// a default plan of at most kFuseMaxSplits splits per head group, which then
// run as one cluster.  (Cutting a longer plan down to that many splits slows
// the reduce by more than the separate combine kernel costs.)
bool fuse_plan(const la::Plan &p) {
    return p.nb == 1 && p.H % 4 == 0 && p.P >= 1 && p.P <= la::kFuseMaxSplits;
}

bool sizes_ok(int B, int N, int H, int d) {
    return B > 0 && N > 0 && H > 0 && d > 0 &&
           (long long)B * N * H * d < (1LL << 40);
}

la_status check_rope(const la_rope *r, int d, bool allow_state_offset) {
    if (!r) return LA_OK;
    if (r->Hg <= 0 || r->Wg <= 0 || r->T < 0) return LA_EINVAL;
    if (r->dt < 0 || r->dh < 0 || r->dw < 0) return LA_EINVAL;
    if ((r->dt | r->dh | r->dw) & 1) return LA_EINVAL;
    if (r->dt + r->dh + r->dw != d) return LA_EINVAL;
    if (!(r->base > 0.0f) || !std::isfinite(r->base)) return LA_EINVAL;
    if (r->t_offset < 0 && !allow_state_offset) return LA_EINVAL;
    return LA_OK;
}

// Frequencies of the 16 feature pairs, computed in double and rounded once.
void fill_rope(la::Plan &p, const la_rope *r, int t_offset) {
    p.rope = r != nullptr;
    p.Hg = r ? r->Hg : 1;
    p.Wg = r ? r->Wg : 1;
    p.t_offset = t_offset;
    la::magic_div((unsigned)((long long)p.Hg * p.Wg < (1LL << 31) ? p.Hg * p.Wg : 0x7fffffff), p.hw_m, p.hw_s);
    la::magic_div((unsigned)p.Wg, p.wg_m, p.wg_s);
    for (int pr = 0; pr < la::kD / 2; ++pr) {
        p.theta[pr] = 0.0f;
        p.axis[pr] = 0;
        if (!r) continue;
        int f = 2 * pr, lo, D, ax;
        if (f < r->dt) { lo = 0; D = r->dt; ax = 0; }
        else if (f < r->dt + r->dh) { lo = r->dt; D = r->dh; ax = 1; }
        else { lo = r->dt + r->dh; D = r->dw; ax = 2; }
        int i = (f - lo) / 2;
        p.theta[pr] = (float)std::pow((double)r->base, -2.0 * (double)i / (double)D);
        p.axis[pr] = ax;
    }
    la::plan_rope_table(p);
}

la_status common_checks(const void *q, const void *k, const void *v, void *out, la_dtype dt,
                        int B, int N, int H, int d, float eps) {
    if (!q || !k || !v || !out) return LA_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_EINVAL;
    if (dt != LA_F32 && dt != LA_BF16) return LA_EINVAL;
    if (!sizes_ok(B, N, H, d)) return LA_EINVAL;
    if (d != la::kD) return LA_EUNSUPPORTED;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return LA_EINVAL;
    return LA_OK;
}

// The tensor-core kernels take bf16 inputs with H a multiple of 4 (4-head
// reduce groups, 2-head apply tiles) and, with RoPE, a cos/sin table that fits
// their shared memory; the rest runs on the CUDA cores.
bool use_tc(la_dtype dt, const la::Plan &p) {
    if (p.f8) return (p.H % 4) == 0 && (!p.rope || la::tc_rope_fits(p)) && la::tc_available();
    if (p.f4) return (p.H % 8) == 0 && (!p.rope || la::tc_rope_fits(p)) && la::tc_available();
    return dt == LA_BF16 && (p.H % 4) == 0 && (!p.rope || la::tc_rope_fits(p)) && la::tc_available();
}

// FP8 E4M3 calls: q, k, v codes with per-tensor scales, bf16 out; tensor cores
// only (H a multiple of 4; with RoPE, a grid whose cos/sin table fits the RoPE
// kernels' shared memory).
la_status e4m3_checks(const void *q, const void *k, const void *v, void *out, int B, int N, int H, int d,
                      float eps, float sq, float sk, float sv) {
    la_status e = common_checks(q, k, v, out, LA_BF16, B, N, H, d, eps);
    if (e != LA_OK) return e;
    for (float x : {sq, sk, sv})
        if (!(x > 0.0f) || !std::isfinite(x)) return LA_EINVAL;
    if (H % 4 != 0 || !la::tc_available()) return LA_EUNSUPPORTED;
    return LA_OK;
}

// NVFP4 calls: q, k, v E2M1 codes [B][N][H][16] bytes, E4M3 block scales
// [B][N][H][2] bytes, per-tensor scales; bf16 out; tensor cores only (H a
// multiple of 8: the scale rows are then whole 16-byte units; with RoPE, a
// grid whose cos/sin table fits the RoPE kernels' shared memory).
la_status nvfp4_checks(const void *q, const void *k, const void *v, const void *sq_blk, const void *sk_blk,
                       const void *sv_blk, void *out, int B, int N, int H, int d, float eps, float sq, float sk,
                       float sv) {
    la_status e = common_checks(q, k, v, out, LA_BF16, B, N, H, d, eps);
    if (e != LA_OK) return e;
    if (!sq_blk || !sk_blk || !sv_blk) return LA_EINVAL;
    if (!aligned16(sq_blk) || !aligned16(sk_blk) || !aligned16(sv_blk)) return LA_EINVAL;
    for (float x : {sq, sk, sv})
        if (!(x > 0.0f) || !std::isfinite(x)) return LA_EINVAL;
    if (H % 8 != 0 || !la::tc_available()) return LA_EUNSUPPORTED;
    return LA_OK;
}

// Enqueue reduce -> finish -> apply for a prepared plan.
la_status run(const void *q, const void *k, const void *v, void *out, la_dtype dt,
              la::Plan &p, float *S, float *Z, void *ws, cudaStream_t s) {
    la::WsLayout w = la::ws_layout(p.B, p.H, p.nb, la::ws_slots(p));
    char *base = static_cast<char *>(ws);
    float *partials = reinterpret_cast<float *>(base + w.partials);
    float *seff = reinterpret_cast<float *>(base + w.seff);
    void *bop = base + w.bop;
    const bool tc = use_tc(dt, p);
    int n = 0, r;

    if (!mark(0, s)) return LA_ECUDA;
    if (tc && p.rope) {
        // RoPE: stream-K reduce, the combine over its slots, stream-K apply
        p.sk_layout = 1;
        r = la::launch_reduce_rope_tc(k, v, partials, p, s);
        if (r < 0 || !mark(1, s)) return LA_ECUDA;
        n += r;
        r = la::launch_finish(partials, seff, bop, S, Z, p, 1, s);
        if (r < 0 || !mark(2, s)) return LA_ECUDA;
        n += r;
        r = la::launch_apply_rope_tc(q, out, bop, seff, p, s);
        if (r < 0 || !mark(3, s)) return LA_ECUDA;
        n += r;
        g_last_launches = n;
        g_last_path = p.f8 ? "tc_e4m3" : (p.f4 ? "tc_nvfp4" : "tc");
        return LA_OK;
    }
    if (tc && fuse_plan(p)) {
        // one block: the reduce combines its splits itself (no combine kernel)
        const la::Fuse fz = {seff, static_cast<unsigned char *>(bop), S, Z, 1, 1};
        r = la::launch_reduce_tc(k, v, partials, p, s, &fz);
        if (r < 0 || !mark(1, s) || !mark(2, s)) return LA_ECUDA;
        n += r;
    } else {
        r = tc ? la::launch_reduce_tc(k, v, partials, p, s)
               : la::launch_reduce_ffma(dt == LA_BF16, k, v, partials, p, s);
        if (r < 0 || !mark(1, s)) return LA_ECUDA;
        n += r;
        r = la::launch_finish(partials, seff, bop, S, Z, p, tc ? 1 : 0, s);
        if (r < 0 || !mark(2, s)) return LA_ECUDA;
        n += r;
    }
    r = tc ? la::launch_apply_tc(q, out, bop, seff, p, s)
           : la::launch_apply_ffma(dt == LA_BF16, q, out, seff, p, s);
    if (r < 0 || !mark(3, s)) return LA_ECUDA;
    n += r;
    g_last_launches = n;
    g_last_path = tc ? (p.f8 ? "tc_e4m3" : (p.f4 ? "tc_nvfp4" : "tc")) : "ffma";
    return LA_OK;
}

}  // namespace

extern "C" {

size_t la_workspace_size(int B, int N, int H, int d, int tokens_per_block) {
    if (!sizes_ok(B, N, H, d) || tokens_per_block < 0) return 0;
    la::Plan p{};
    p.B = B; p.N = N; p.H = H;
    p.L = tokens_per_block > 0 && tokens_per_block < N ? tokens_per_block : N;
    p.nb = (int)ceil_div(N, p.L);
    make_splits(p);
    return la::ws_layout(B, H, p.nb, la::ws_slots(p)).total;
}

la_status la_state_init(la_state *st, float *S, float *Z, int B, int H, int d, void *stream) {
    if (!st || !S || !Z) return LA_EINVAL;
    if (B <= 0 || H <= 0 || d <= 0) return LA_EINVAL;
    if (d != la::kD) return LA_EUNSUPPORTED;
    if (!aligned16(S) || !aligned16(Z)) return LA_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t nS = size_t(B) * H * d * d, nZ = size_t(B) * H * d;
    if (cudaMemsetAsync(S, 0, nS * sizeof(float), s) != cudaSuccess) return LA_ECUDA;
    if (cudaMemsetAsync(Z, 0, nZ * sizeof(float), s) != cudaSuccess) return LA_ECUDA;
    st->S = S; st->Z = Z; st->B = B; st->H = H; st->d = d;
    st->blocks_committed = 0;
    st->t_next = 0;
    return LA_OK;
}

// A bound state: what la_state_init leaves behind.
static bool state_bound(const la_state *st) {
    return st && st->S && st->Z && st->B > 0 && st->H > 0 && st->d == la::kD;
}

la_status la_state_save(const la_state *st, float *S_dst, float *Z_dst, la_state_counters *counters,
                        void *stream) {
    if (!state_bound(st) || !S_dst || !Z_dst || !counters) return LA_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t nS = size_t(st->B) * st->H * st->d * st->d, nZ = size_t(st->B) * st->H * st->d;
    if (cudaMemcpyAsync(S_dst, st->S, nS * sizeof(float), cudaMemcpyDefault, s) != cudaSuccess) return LA_ECUDA;
    if (cudaMemcpyAsync(Z_dst, st->Z, nZ * sizeof(float), cudaMemcpyDefault, s) != cudaSuccess) return LA_ECUDA;
    counters->blocks_committed = st->blocks_committed;
    counters->t_next = st->t_next;
    return LA_OK;
}

la_status la_state_restore(la_state *st, const float *S_src, const float *Z_src,
                           const la_state_counters *counters, void *stream) {
    if (!state_bound(st) || !S_src || !Z_src || !counters) return LA_EINVAL;
    if (counters->blocks_committed < 0 || counters->t_next < 0) return LA_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t nS = size_t(st->B) * st->H * st->d * st->d, nZ = size_t(st->B) * st->H * st->d;
    if (cudaMemcpyAsync(st->S, S_src, nS * sizeof(float), cudaMemcpyDefault, s) != cudaSuccess) return LA_ECUDA;
    if (cudaMemcpyAsync(st->Z, Z_src, nZ * sizeof(float), cudaMemcpyDefault, s) != cudaSuccess) return LA_ECUDA;
    st->blocks_committed = counters->blocks_committed;
    st->t_next = counters->t_next;
    return LA_OK;
}

la_status la_block_forward(const void *q, const void *k, const void *v, void *out, la_dtype dt,
                           int B, int N_blk, int H, int d, la_state *st, int commit,
                           const la_rope *rope, float eps, void *ws, size_t ws_bytes,
                           void *stream) {
    la_status e = common_checks(q, k, v, out, dt, B, N_blk, H, d, eps);
    if (e != LA_OK) return e;
    if (!st || !st->S || !st->Z) return LA_EINVAL;
    if (st->B != B || st->H != H || st->d != d) return LA_EINVAL;
    if ((e = check_rope(rope, d, true)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N_blk, H, d, N_blk);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;

    la::Plan p{};
    p.B = B; p.N = N_blk; p.H = H; p.L = N_blk; p.nb = 1;
    p.commit = commit != 0;
    p.has_state = 1;
    p.eps = eps;
    make_splits(p);
    fill_rope(p, rope, rope ? (rope->t_offset < 0 ? st->t_next : rope->t_offset) : 0);
    e = run(q, k, v, out, dt, p, st->S, st->Z, ws, static_cast<cudaStream_t>(stream));
    if (e != LA_OK) return e;
    if (commit) {
        st->blocks_committed += 1;
        if (rope) st->t_next += rope->T;
    }
    return LA_OK;
}

la_status la_full_forward(const void *q, const void *k, const void *v, void *out, la_dtype dt,
                          int B, int N, int H, int d, int tokens_per_block,
                          const la_rope *rope, float eps, void *ws, size_t ws_bytes,
                          void *stream) {
    la_status e = common_checks(q, k, v, out, dt, B, N, H, d, eps);
    if (e != LA_OK) return e;
    if (tokens_per_block < 0) return LA_EINVAL;
    if ((e = check_rope(rope, d, false)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N, H, d, tokens_per_block);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;

    la::Plan p{};
    p.B = B; p.N = N; p.H = H;
    p.L = tokens_per_block > 0 && tokens_per_block < N ? tokens_per_block : N;
    p.nb = (int)ceil_div(N, p.L);
    p.commit = 0;
    p.has_state = 0;
    p.eps = eps;
    make_splits(p);
    fill_rope(p, rope, rope ? rope->t_offset : 0);
    return run(q, k, v, out, dt, p, nullptr, nullptr, ws, static_cast<cudaStream_t>(stream));
}

size_t la_backward_workspace_size(int B, int N, int H, int d, int tokens_per_block) {
    if (!sizes_ok(B, N, H, d) || tokens_per_block < 0) return 0;
    la::Plan p{};
    p.B = B; p.N = N; p.H = H;
    p.L = tokens_per_block > 0 && tokens_per_block < N ? tokens_per_block : N;
    p.nb = (int)ceil_div(N, p.L);
    make_splits(p);
    return la::bwd_layout(B, H, p.nb, la::ws_slots(p)).total;
}

la_status la_full_backward(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                           void *dv, la_dtype dt, int B, int N, int H, int d, int tokens_per_block,
                           const la_rope *rope, float eps, void *ws, size_t ws_bytes, void *stream) {
    la_status e = common_checks(q, k, v, dq, dt, B, N, H, d, eps);
    if (e != LA_OK) return e;
    if (!dout || !dk || !dv || !aligned16(dout) || !aligned16(dk) || !aligned16(dv)) return LA_EINVAL;
    if (tokens_per_block < 0) return LA_EINVAL;
    if ((e = check_rope(rope, d, false)) != LA_OK) return e;
    const size_t need = la_backward_workspace_size(B, N, H, d, tokens_per_block);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;

    la::Plan p{};
    p.B = B; p.N = N; p.H = H;
    p.L = tokens_per_block > 0 && tokens_per_block < N ? tokens_per_block : N;
    p.nb = (int)ceil_div(N, p.L);
    p.commit = 0;
    p.has_state = 0;
    p.eps = eps;
    make_splits(p);
    fill_rope(p, rope, rope ? rope->t_offset : 0);

    const la::BwdLayout w = la::bwd_layout(B, H, p.nb, la::ws_slots(p));
    char *base = static_cast<char *>(ws);
    float *partials = reinterpret_cast<float *>(base + w.fwd.partials);
    float *seff = reinterpret_cast<float *>(base + w.fwd.seff);
    float *bpart = reinterpret_cast<float *>(base + w.bpart);
    float *G = reinterpret_cast<float *>(base + w.G);
    void *gop = base + w.gop;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool tc = use_tc(dt, p);
    const int bf = dt == LA_BF16;
    int n = 0, r;
    // stage events (la_set_stage_events): before the state pass, after it,
    // after the query side, after the key side
    if (!mark(0, s)) return LA_ECUDA;
    // the forward prefix state S_n, Z_n of every block, as the forward computes it
    if (tc && p.rope) p.sk_layout = 1;
    r = tc ? (p.rope ? la::launch_reduce_rope_tc(k, v, partials, p, s) : la::launch_reduce_tc(k, v, partials, p, s))
           : la::launch_reduce_ffma(bf, k, v, partials, p, s);
    if (r < 0) return LA_ECUDA;
    n += r;
    // the query side on the tensor cores needs the packed [S|Z|0] operand
    const bool qtc = bf && tc && la::bwd_q_tc_available(p);
    r = la::launch_finish(partials, seff, base + w.fwd.bop, nullptr, nullptr, p, tc ? 1 : 0, s);
    if (r < 0) return LA_ECUDA;
    n += r;
    if (!mark(1, s)) return LA_ECUDA;
    // the query side takes its own split plan; the suffix sums below read its splits
    la::Plan pq = p;
    if (qtc) la::bwd_q_tc_plan(pq);
    r = qtc ? la::launch_bwd_q_tc(q, dout, dq, seff, base + w.fwd.bop, bpart, pq, s)
            : la::launch_bwd_q(bf, q, dout, seff, dq, bpart, p, s);
    if (r < 0) return LA_ECUDA;
    n += r;
    if (!mark(2, s)) return LA_ECUDA;
    const bool ktc = bf && la::bwd_k_tc_available(p);
    if ((r = la::launch_bwd_finish(bpart, G, ktc ? gop : nullptr, qtc ? pq : p, s)) < 0) return LA_ECUDA;
    n += r;
    r = ktc ? la::launch_bwd_k_tc(k, v, G, gop, dk, dv, p, s) : la::launch_bwd_k(bf, k, v, G, dk, dv, p, s);
    if (r < 0) return LA_ECUDA;
    n += r;
    if (!mark(3, s)) return LA_ECUDA;
    g_last_launches = n;
    g_last_path = qtc && ktc ? "bwd_tc" : (ktc ? "bwd(tc state, tc keys)" : (tc ? "bwd(tc state)" : "bwd"));
    return LA_OK;
}

la_status la_full_forward_e4m3(const void *q, const void *k, const void *v, float scale_q, float scale_k,
                               float scale_v, void *out, int B, int N, int H, int d, int tokens_per_block,
                               const la_rope *rope, float eps, void *ws, size_t ws_bytes, void *stream) {
    la_status e = e4m3_checks(q, k, v, out, B, N, H, d, eps, scale_q, scale_k, scale_v);
    if (e != LA_OK) return e;
    if (tokens_per_block < 0) return LA_EINVAL;
    if ((e = check_rope(rope, d, false)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N, H, d, tokens_per_block);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;
    la::Plan p{};
    p.B = B; p.N = N; p.H = H;
    p.L = tokens_per_block > 0 && tokens_per_block < N ? tokens_per_block : N;
    p.nb = (int)ceil_div(N, p.L);
    p.eps = eps;
    p.f8 = 1;
    p.sq = scale_q; p.sk = scale_k; p.sv = scale_v;
    make_splits(p);
    fill_rope(p, rope, rope ? rope->t_offset : 0);
    if (!use_tc(LA_BF16, p)) return LA_EUNSUPPORTED;   // E4M3 runs on the tensor cores only
    return run(q, k, v, out, LA_BF16, p, nullptr, nullptr, ws, static_cast<cudaStream_t>(stream));
}

la_status la_block_forward_e4m3(const void *q, const void *k, const void *v, float scale_q, float scale_k,
                                float scale_v, void *out, int B, int N_blk, int H, int d, la_state *st, int commit,
                                const la_rope *rope, float eps, void *ws, size_t ws_bytes, void *stream) {
    la_status e = e4m3_checks(q, k, v, out, B, N_blk, H, d, eps, scale_q, scale_k, scale_v);
    if (e != LA_OK) return e;
    if (!st || !st->S || !st->Z) return LA_EINVAL;
    if (st->B != B || st->H != H || st->d != d) return LA_EINVAL;
    if ((e = check_rope(rope, d, true)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N_blk, H, d, N_blk);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;
    la::Plan p{};
    p.B = B; p.N = N_blk; p.H = H; p.L = N_blk; p.nb = 1;
    p.commit = commit != 0;
    p.has_state = 1;
    p.eps = eps;
    p.f8 = 1;
    p.sq = scale_q; p.sk = scale_k; p.sv = scale_v;
    make_splits(p);
    fill_rope(p, rope, rope ? (rope->t_offset < 0 ? st->t_next : rope->t_offset) : 0);
    if (!use_tc(LA_BF16, p)) return LA_EUNSUPPORTED;   // E4M3 runs on the tensor cores only
    e = run(q, k, v, out, LA_BF16, p, st->S, st->Z, ws, static_cast<cudaStream_t>(stream));
    if (e != LA_OK) return e;
    if (commit) {
        st->blocks_committed += 1;
        if (rope) st->t_next += rope->T;
    }
    return LA_OK;
}

la_status la_full_forward_nvfp4(const void *q, const void *k, const void *v, const void *q_blk_scale,
                                const void *k_blk_scale, const void *v_blk_scale, float scale_q, float scale_k,
                                float scale_v, void *out, int B, int N, int H, int d, int tokens_per_block,
                                const la_rope *rope, float eps, void *ws, size_t ws_bytes, void *stream) {
    la_status e = nvfp4_checks(q, k, v, q_blk_scale, k_blk_scale, v_blk_scale, out, B, N, H, d, eps, scale_q,
                               scale_k, scale_v);
    if (e != LA_OK) return e;
    if (tokens_per_block < 0) return LA_EINVAL;
    if ((e = check_rope(rope, d, false)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N, H, d, tokens_per_block);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;
    la::Plan p{};
    p.B = B; p.N = N; p.H = H;
    p.L = tokens_per_block > 0 && tokens_per_block < N ? tokens_per_block : N;
    p.nb = (int)ceil_div(N, p.L);
    p.eps = eps;
    p.f4 = 1;
    p.sq = scale_q; p.sk = scale_k; p.sv = scale_v;
    p.sfq = q_blk_scale; p.sfk = k_blk_scale; p.sfv = v_blk_scale;
    make_splits(p);
    fill_rope(p, rope, rope ? rope->t_offset : 0);
    if (!use_tc(LA_BF16, p)) return LA_EUNSUPPORTED;   // NVFP4 runs on the tensor cores only
    return run(q, k, v, out, LA_BF16, p, nullptr, nullptr, ws, static_cast<cudaStream_t>(stream));
}

la_status la_block_forward_nvfp4(const void *q, const void *k, const void *v, const void *q_blk_scale,
                                 const void *k_blk_scale, const void *v_blk_scale, float scale_q, float scale_k,
                                 float scale_v, void *out, int B, int N_blk, int H, int d, la_state *st, int commit,
                                 const la_rope *rope, float eps, void *ws, size_t ws_bytes, void *stream) {
    la_status e = nvfp4_checks(q, k, v, q_blk_scale, k_blk_scale, v_blk_scale, out, B, N_blk, H, d, eps, scale_q,
                               scale_k, scale_v);
    if (e != LA_OK) return e;
    if (!st || !st->S || !st->Z) return LA_EINVAL;
    if (st->B != B || st->H != H || st->d != d) return LA_EINVAL;
    if ((e = check_rope(rope, d, true)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N_blk, H, d, N_blk);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;
    la::Plan p{};
    p.B = B; p.N = N_blk; p.H = H; p.L = N_blk; p.nb = 1;
    p.commit = commit != 0;
    p.has_state = 1;
    p.eps = eps;
    p.f4 = 1;
    p.sq = scale_q; p.sk = scale_k; p.sv = scale_v;
    p.sfq = q_blk_scale; p.sfk = k_blk_scale; p.sfv = v_blk_scale;
    make_splits(p);
    fill_rope(p, rope, rope ? (rope->t_offset < 0 ? st->t_next : rope->t_offset) : 0);
    if (!use_tc(LA_BF16, p)) return LA_EUNSUPPORTED;   // NVFP4 runs on the tensor cores only
    e = run(q, k, v, out, LA_BF16, p, st->S, st->Z, ws, static_cast<cudaStream_t>(stream));
    if (e != LA_OK) return e;
    if (commit) {
        st->blocks_committed += 1;
        if (rope) st->t_next += rope->T;
    }
    return LA_OK;
}

la_status la_dwconv3d(const void *x, void *y, la_dtype dt, int B, int T, int Hg, int Wg, int C, int kt, int kh,
                      int kw, const float *weight, const float *bias, void *stream) {
    if (!x || !y || !weight || !aligned16(x) || !aligned16(y)) return LA_EINVAL;
    if (dt != LA_F32 && dt != LA_BF16) return LA_EINVAL;
    if (B <= 0 || T <= 0 || Hg <= 0 || Wg <= 0 || C <= 0) return LA_EINVAL;
    if ((long long)B * T * Hg * Wg * C >= (1LL << 40)) return LA_EINVAL;
    if (C % 8 != 0) return LA_EUNSUPPORTED;
    const int r = la::launch_dwconv(dt == LA_BF16, x, y, weight, bias, B, T, Hg, Wg, C, kt, kh, kw,
                                    static_cast<cudaStream_t>(stream));
    if (r == -2) return LA_EUNSUPPORTED;
    if (r < 0) return LA_ECUDA;
    g_last_launches = r;
    g_last_path = "dwconv";
    return LA_OK;
}

size_t la_split_partial_bytes(int B, int H, int d) {
    if (B <= 0 || H <= 0 || d != la::kD) return 0;
    return size_t(B) * H * la::kKVZ * sizeof(float);
}

la_status la_block_reduce(const void *k, const void *v, la_dtype dt, int B, int N_slice, int H, int d,
                          const la_rope *rope, float *partial, void *ws, size_t ws_bytes, void *stream) {
    la_status e = common_checks(k, k, v, partial, dt, B, N_slice, H, d, 0.0f);
    if (e != LA_OK) return e;
    if ((e = check_rope(rope, d, false)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N_slice, H, d, N_slice);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;
    la::Plan p{};
    p.B = B; p.N = N_slice; p.H = H; p.L = N_slice; p.nb = 1;
    make_splits(p);
    fill_rope(p, rope, rope ? rope->t_offset : 0);
    const la::WsLayout w = la::ws_layout(B, H, 1, la::ws_slots(p));
    char *base = static_cast<char *>(ws);
    float *partials = reinterpret_cast<float *>(base + w.partials);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool tc = use_tc(dt, p);
    int n = 0, r;
    if (tc && p.rope) p.sk_layout = 1;
    r = tc ? (p.rope ? la::launch_reduce_rope_tc(k, v, partials, p, s) : la::launch_reduce_tc(k, v, partials, p, s))
           : la::launch_reduce_ffma(dt == LA_BF16, k, v, partials, p, s);
    if (r < 0) return LA_ECUDA;
    n += r;
    // the slice's split sums, in split order, straight into the caller's partial
    if ((r = la::launch_finish(partials, partial, base + w.bop, nullptr, nullptr, p, 0, s)) < 0) return LA_ECUDA;
    n += r;
    g_last_launches = n;
    g_last_path = tc ? "tc" : "ffma";
    return LA_OK;
}

la_status la_block_apply(const void *q, void *out, la_dtype dt, int B, int N_slice, int H, int d,
                         const float *gathered, int R, la_state *st, int commit, const la_rope *rope, float eps,
                         void *ws, size_t ws_bytes, void *stream) {
    la_status e = common_checks(q, q, q, out, dt, B, N_slice, H, d, eps);
    if (e != LA_OK) return e;
    if (!gathered || !aligned16(gathered) || R < 1 || R > 32) return LA_EINVAL;
    if (!st || !st->S || !st->Z || st->B != B || st->H != H || st->d != d) return LA_EINVAL;
    if ((e = check_rope(rope, d, true)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N_slice, H, d, N_slice);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return LA_EWORKSPACE;
    la::Plan p{};
    p.B = B; p.N = N_slice; p.H = H; p.L = N_slice; p.nb = 1;
    p.commit = commit != 0;
    p.has_state = 1;
    p.eps = eps;
    make_splits(p);
    fill_rope(p, rope, rope ? (rope->t_offset < 0 ? st->t_next : rope->t_offset) : 0);
    const la::WsLayout w = la::ws_layout(B, H, 1, la::ws_slots(p));
    char *base = static_cast<char *>(ws);
    float *seff = reinterpret_cast<float *>(base + w.seff);
    void *bop = base + w.bop;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool tc = use_tc(dt, p);
    int n = 0, r;
    if ((r = la::launch_finish_ranks(gathered, R, seff, bop, st->S, st->Z, p, tc ? 1 : 0, s)) < 0) return LA_ECUDA;
    n += r;
    r = tc ? (p.rope ? la::launch_apply_rope_tc(q, out, bop, seff, p, s) : la::launch_apply_tc(q, out, bop, seff, p, s))
           : la::launch_apply_ffma(dt == LA_BF16, q, out, seff, p, s);
    if (r < 0) return LA_ECUDA;
    n += r;
    g_last_launches = n;
    g_last_path = tc ? "tc" : "ffma";
    if (commit) {
        st->blocks_committed += 1;
        if (rope) st->t_next += rope->T;
    }
    return LA_OK;
}

la_status la_device_status(void *stream) {
    unsigned flag = 0, fk = 0, fq = 0, fc = 0, fr = 0;
    // (synchronises the stream first)
    if (la::read_and_clear_device_flag(static_cast<cudaStream_t>(stream), &flag) != 0) return LA_ECUDA;
    if (la::read_and_clear_bwd_k_flag(&fk) != 0 || la::read_and_clear_bwd_q_flag(&fq) != 0 ||
        la::read_and_clear_conv_flag(&fc) != 0 || la::read_and_clear_rope_flag(&fr) != 0)
        return LA_ECUDA;
    return (flag | fk | fq | fc | fr) ? LA_ETIMEOUT : LA_OK;
}

la_status la_selftest_bounded_wait(void *stream) {
    return la::launch_bounded_wait_selftest(static_cast<cudaStream_t>(stream)) < 0 ? LA_ECUDA : LA_OK;
}

const char *la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_EINVAL: return "LA_EINVAL: invalid argument";
        case LA_EUNSUPPORTED: return "LA_EUNSUPPORTED: unsupported shape (d must be 32)";
        case LA_ECUDA: return "LA_ECUDA: CUDA call or kernel launch failed";
        case LA_ETIMEOUT: return "LA_ETIMEOUT: a device-side bounded wait gave up";
        case LA_EWORKSPACE: return "LA_EWORKSPACE: workspace missing, misaligned or too small";
    }
    return "LA_?: unknown status";
}

void la_set_stage_events(void *before_reduce, void *after_reduce, void *after_finish,
                         void *after_apply) {
    g_ev[0] = static_cast<cudaEvent_t>(before_reduce);
    g_ev[1] = static_cast<cudaEvent_t>(after_reduce);
    g_ev[2] = static_cast<cudaEvent_t>(after_finish);
    g_ev[3] = static_cast<cudaEvent_t>(after_apply);
}

int la_last_launch_count(void) { return g_last_launches; }

int la_tc_enabled(void) { return la::tc_available() ? 1 : 0; }

const char *la_last_path(void) { return g_last_path; }

}  // extern "C"

// ---------------------------------------------------------------- static scratch
// la_full_forward_static_ws: la_full_forward with its workspace in a file-scope
// device array, for callers that cannot allocate.  In host code the array's
// name only stands for the symbol; its device address comes from
// cudaGetSymbolAddress, once per device, with that device current.
static __device__ __align__(256) unsigned char g_la_static_ws[LA_STATIC_WS_BYTES];

namespace {
constexpr int kMaxDevices = 128;
void *g_static_ws_ptr[kMaxDevices] = {};
std::mutex g_static_ws_mutex;

la_status static_ws_for_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LA_ECUDA;
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    if (!g_static_ws_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_la_static_ws) != cudaSuccess || !p) return LA_ECUDA;
        g_static_ws_ptr[dev] = p;
    }
    *out = g_static_ws_ptr[dev];
    return LA_OK;
}
}  // namespace

extern "C" la_status la_full_forward_static_ws(const void *q, const void *k, const void *v, void *out,
                                               la_dtype dt, int B, int N, int H, int d,
                                               int tokens_per_block, const la_rope *rope, float eps,
                                               void *stream) {
    la_status e = common_checks(q, k, v, out, dt, B, N, H, d, eps);
    if (e != LA_OK) return e;
    if (tokens_per_block < 0) return LA_EINVAL;
    if ((e = check_rope(rope, d, false)) != LA_OK) return e;
    const size_t need = la_workspace_size(B, N, H, d, tokens_per_block);
    if (need == 0 || need > LA_STATIC_WS_BYTES) return LA_EWORKSPACE;
    void *ws = nullptr;
    if ((e = static_ws_for_current_device(&ws)) != LA_OK) return e;
    return la_full_forward(q, k, v, out, dt, B, N, H, d, tokens_per_block, rope, eps, ws,
                           LA_STATIC_WS_BYTES, stream);
}
