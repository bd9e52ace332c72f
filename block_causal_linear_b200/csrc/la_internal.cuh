// la_internal.cuh -- shared host/device declarations of libla_b200.so.
//
// The launch plan, the workspace layout and the kernel launchers that
// la_api.cu calls.  Nothing here is part of the public ABI (include/la.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <utility>

namespace la {

constexpr int kD = 32;                 // head dim supported by this build
constexpr int kKVZ = kD * kD + kD;     // floats per (b, h) of [KV | z]: KV[dk][dv] then z[dk]
constexpr int kSmCount = 148;          // SMs of a B200
constexpr int kTargetCtas = 296;       // 2 resident CTAs on each of the 148 SMs of a B200
constexpr int kReduceRows = 64;        // token rows per reduce pipeline stage
constexpr int kApplyRows = 128;        // token rows per apply tile (= MMA M)
constexpr int kOpRows = 48;            // N of the apply MMA: 32 S columns, Z, 15 zero rows
constexpr int kOpBytes = kOpRows * kD * 2;   // one bf16 operand (hi or lo) = 3072 B

// A stream-K plan: a call's work as units (a head group or a head pair of one
// batch element and block) in the order (b, block, unit), each unit cut into
// granules of a fixed number of tokens; CTA c takes granules
// [c * total / C, (c + 1) * total / C) of that order, so every CTA gets the
// same amount of work whatever the shapes.  A function of the shapes only.
struct Sk {
    long long total;   // granules in the call
    int C;             // CTAs
    int units;         // units per (b, block)
    int g_full;        // granules of a full block
    int g_last;        // granules of the last block
    int nb;            // blocks
};

__host__ __device__ inline long long sk_per_b(const Sk &s) {
    return (long long)s.units * ((long long)(s.nb - 1) * s.g_full + s.g_last);
}
// First granule of CTA c (c = C gives the end).
__host__ __device__ inline long long sk_cta_start(const Sk &s, int c) { return (long long)c * s.total / s.C; }
// The CTA whose range holds granule x.
__host__ __device__ inline int sk_cta_of(const Sk &s, long long x) {
    return (int)(((x + 1) * (long long)s.C - 1) / s.total);
}
// Granules of a unit of block n, and the first granule of unit (b, n, u).
__host__ __device__ inline int sk_len(const Sk &s, int n) { return n < s.nb - 1 ? s.g_full : s.g_last; }
__host__ __device__ inline long long sk_unit_first(const Sk &s, int b, int n, int u) {
    return (long long)b * sk_per_b(s) + (long long)n * s.units * s.g_full + (long long)u * sk_len(s, n);
}
// The unit (b, n, u) that holds granule x.
__host__ __device__ inline void sk_locate(const Sk &s, long long x, int &b, int &n, int &u) {
    const long long pb = sk_per_b(s);
    b = (int)(x / pb);
    long long r = x - (long long)b * pb;
    const long long full = (long long)(s.nb - 1) * s.units * s.g_full;
    if (r < full) {
        const long long blk = (long long)s.units * s.g_full;
        n = (int)(r / blk);
        r -= (long long)n * blk;
        u = (int)(r / s.g_full);
    } else {
        n = s.nb - 1;
        u = (int)((r - full) / s.g_last);
    }
}

// Everything a kernel needs to know about one call, passed by value.
// Input kinds of the tensor-core kernels: bf16 q, k, v; FP8 E4M3 codes with
// per-tensor scales; NVFP4 (E2M1 codes, an E4M3 scale per 16 features, a
// per-tensor scale).
constexpr int kInBf16 = 0, kInE4m3 = 1, kInNvfp4 = 2;

struct Plan {
    int B, N, H;          // batch, tokens in the call, heads
    int L;                // tokens per block (the last block may be shorter)
    int nb;               // number of blocks in the call
    int P;                // reduce splits per (b, h, block)
    int chunk;            // tokens per reduce split (multiple of 16)
    int Pa;               // apply splits per (b, head pair, block)
    int chunka;           // tokens per apply split (multiple of kApplyRows)
    int commit;           // write S_eff of the last block back to the state
    int has_state;        // S, Z hold a prior state (block_forward) or not (full_forward)
    int rope;             // numerator RoPE on phi(q), phi(k)
    int f8;               // q, k, v are FP8 E4M3 codes with per-tensor scales sq, sk, sv
    int f4;               // q, k, v are NVFP4: E2M1 codes, E4M3 block scales sfq, sfk, sfv, per-tensor sq, sk, sv
    float sq, sk, sv;
    const void *sfq, *sfk, *sfv;   // NVFP4 block scales [B][N][H][2] (host-side, for the tensor maps)
    int Hg, Wg;           // latent grid of one frame
    int t_offset;         // frame of token 0 of the call
    float eps;
    float theta[kD / 2];  // RoPE frequency of feature pair p
    int axis[kD / 2];     // 0: frame, 1: row, 2: column
    // n / (Hg*Wg) and n / Wg for 0 <= n < 2^31 as (n * m) >> s (division by an
    // invariant integer through a multiply, Granlund & Montgomery 1994)
    unsigned long long hw_m, wg_m;
    int hw_s, wg_s;
    // The RoPE tensor-core kernels (k_rope_tc.cu): stream-K plans of the
    // reduce (head groups x 16-token granules) and of the apply (head pairs x
    // 128-token tiles); the reduce's split sums then sit in skP slots per
    // (b, h, block), slot j holding the sums of the j-th CTA that met the unit.
    int sk_layout;        // the split sums are in the stream-K layout
    int skP;              // slots per (b, h, block) of that layout (a bound)
    Sk skr, ska;
    // Their cos/sin table: the 8 groups of 4 features ("half chunks": 2 pairs
    // each, one axis) read records of (cos a, cos b, sin a, sin b) at byte
    // hc_base[m] + position * hc_stride[m] of the table, position along axis
    // hc_axis[m] (0 frame relative to token 0 of the call, 1 row, 2 column).
    int hc_base[8], hc_stride[8], hc_axis[8];
    int tab_frames;       // frames the table covers (all frames of the call)
    int tab_bytes;        // table size; 0 if the RoPE sections do not fit this layout
};

// m, s with floor(n / d) == (n * m) >> s for every 0 <= n < 2^31 (1 <= d < 2^31):
// l = ceil(log2 d), s = 31 + l, m = ceil(2^s / d); then 2^s <= m d < 2^s + 2^l.
inline void magic_div(unsigned d, unsigned long long &m, int &s) {
    int l = 0;
    while ((1ull << l) < d) ++l;
    s = 31 + l;
    m = ((1ull << s) + d - 1) / d;
}

#ifdef __CUDACC__
__device__ __forceinline__ int fast_div(int n, unsigned long long m, int s) {
    return (int)(((unsigned long long)(unsigned)n * m) >> s);
}

// Byte offset of element (n, k) of one packed bf16 MMA operand [S | Z | 0]
// (K = 32 key features, N = 48 columns): K-major, no swizzle, core matrices
// of 8 rows x 16 bytes, 128 B apart along K and 512 B apart along N.
__device__ __forceinline__ int op_offset(int nrow, int kcol) {
    return (nrow >> 3) * 512 + (kcol >> 3) * 128 + (nrow & 7) * 16 + (kcol & 7) * 2;
}
#endif

// Workspace layout (byte offsets from the 256-byte aligned base).
struct WsLayout {
    size_t partials;      // float [B][H][nb][P][kKVZ]
    size_t seff;          // float [B][H][nb][kKVZ]  effective state S + sum of KV, Z + sum of z
    size_t bop;           // bf16  [B][H][nb][2][kOpRows][kD] packed MMA operand (hi, lo)
    size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Split-sum slots per (b, h, block) that the workspace holds for a plan: the
// split plan's P, or the stream-K layout's, whichever is larger.
inline int ws_slots(const Plan &p) { return p.P > p.skP ? p.P : p.skP; }

inline WsLayout ws_layout(int B, int H, int nb, int P) {
    WsLayout w;
    size_t bhn = size_t(B) * H * nb;
    w.partials = 0;
    w.seff = align256(w.partials + bhn * P * kKVZ * sizeof(float));
    w.bop = align256(w.seff + bhn * kKVZ * sizeof(float));
    w.total = align256(w.bop + bhn * 2 * size_t(kOpBytes));
    return w;
}

// ---------------------------------------------------------------- launchers
// Each returns the number of kernels enqueued (>= 0) or -1 on a launch error.

// fp32/bf16 CUDA-core path (any H).  T is float or __nv_bfloat16.
int launch_reduce_ffma(int is_bf16, const void *k, const void *v, float *partials,
                       const Plan &p, cudaStream_t s);
int launch_apply_ffma(int is_bf16, const void *q, void *out, const float *seff,
                      const Plan &p, cudaStream_t s);

// Fixed-order sum of the split partials, prefix over blocks, + prior state;
// writes S_eff (fp32), the packed bf16 hi/lo tensor-core operand, and on
// commit the state.
int launch_finish(const float *partials, float *seff, void *bop, float *S, float *Z,
                  const Plan &p, int write_bop, cudaStream_t s);

// The same, also packing S^T (hi, lo) for the query-side backward; no state.

// The same for a block whose tokens were split over R ranks: gathered is
// [R][B][H][kKVZ], the ranks' partial sums in rank order; p.nb must be 1.
int launch_finish_ranks(const float *gathered, int R, float *seff, void *bop, float *S, float *Z, const Plan &p,
                        int write_bop, cudaStream_t s);

// Tensor-core path (bf16, H % 4 == 0): tcgen05 MMAs, TMA tiles.
// The three kernels of a call (reduce, finish above, apply) order themselves
// by grid through programmatic dependent launch.
// The state combine done by the reduce itself (one block per call, P <= 8):
// the P splits of a head group run as one cluster, add their split sums
// through distributed shared memory in split order, and write S_eff, the
// packed operand and (commit) the state, as launch_finish does.
struct Fuse {
    float *seff;
    unsigned char *bop;
    float *S, *Z;
    int on, write_bop;
};
constexpr int kFuseMaxSplits = 8;
int launch_reduce_tc(const void *k, const void *v, float *partials, const Plan &p, cudaStream_t s,
                     const Fuse *fz = nullptr);
int launch_apply_tc(const void *q, void *out, const void *bop, const float *seff, const Plan &p,
                    cudaStream_t s);
bool tc_available();
// RoPE on the tensor cores (k_rope_tc.cu): the stream-K plans of a call and
// the layout of its cos/sin table (shape-only; sets skr, ska, skP and the
// table fields), whether the table fits the kernels' shared memory, and the
// two kernels.  The reduce writes its split sums in the stream-K layout
// (p.sk must be set for the combine), the apply reads the packed operand and
// Z_eff the combine wrote.
void plan_rope_sk(Plan &p);
void plan_rope_table(Plan &p);
bool tc_rope_fits(const Plan &p);
int launch_reduce_rope_tc(const void *k, const void *v, float *partials, const Plan &p, cudaStream_t s);
int launch_apply_rope_tc(const void *q, void *out, const void *bop, const float *seff, const Plan &p,
                         cudaStream_t s);
int read_and_clear_rope_flag(unsigned *flag_out);

// Backward pass (CUDA cores, fp32 or bf16 tensors): dq and the per-split
// [dS | dZ] sums from q, dout and the forward prefix state; the suffix sums
// over blocks; dk and dv from k, v and those sums.
int launch_bwd_q(int is_bf16, const void *q, const void *dout, const float *seff, void *dq, float *bpart,
                 const Plan &p, cudaStream_t s);
int launch_bwd_finish(const float *bpart, float *G, void *gop, const Plan &p, cudaStream_t s);
// Key side on the tensor cores (bf16, H % 4 == 0; with RoPE when the call's
// cos/sin table fits): dk, dv from k, v and the packed G operands; Gz from G.
bool bwd_k_tc_available(const Plan &p);
int launch_bwd_k_tc(const void *k, const void *v, const float *G, const void *gop, void *dk, void *dv,
                    const Plan &p, cudaStream_t s);
int launch_bwd_k(int is_bf16, const void *k, const void *v, const float *G, void *dk, void *dv, const Plan &p,
                 cudaStream_t s);

// Backward workspace: the forward layout, then the split sums of [dS | dZ]
// ([B][H][nb][P][kKVZ]) and their suffix sums G ([B][H][nb][kKVZ]), fp32.
struct BwdLayout {
    WsLayout fwd;
    size_t bpart, G, gop, total;
};

// Packed bf16 operands of the key-side tensor-core backward, per (b, h,
// block): G (rows = value column c, K = key feature a) and G^T (rows = a,
// K = c), each as a hi and a lo part, 32 rows of the K-major core-matrix
// layout of op_offset: 4 x 2048 bytes.
constexpr int kGopBytes = 2048;

inline BwdLayout bwd_layout(int B, int H, int nb, int P) {
    BwdLayout w;
    w.fwd = ws_layout(B, H, nb, P);
    const size_t bhn = size_t(B) * H * nb;
    w.bpart = w.fwd.total;
    w.G = align256(w.bpart + bhn * P * kKVZ * sizeof(float));
    w.gop = align256(w.G + bhn * kKVZ * sizeof(float));
    w.total = align256(w.gop + bhn * 4 * size_t(kGopBytes));
    return w;
}

// Depthwise 3D convolution (Mix-FFN), kernel shapes 1x3x3 and 3x1x1; returns
// -2 for any other shape.
int launch_dwconv(int is_bf16, const void *x, void *y, const float *w, const float *bias, int B, int T, int Hg,
                  int Wg, int C, int kt, int kh, int kw, cudaStream_t s);

// Launch with programmatic stream serialization (the kernel may start while
// the previous kernel of the stream drains; it orders itself with pdl_wait).
template <typename... KArgs, typename... Args>
bool launch_pdl(void (*kernel)(KArgs...), unsigned grid, int threads, int smem, cudaStream_t s,
                Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess;
}

// The same, launched as clusters of `cluster` consecutive CTAs (portable sizes: <= 8).
template <typename... KArgs, typename... Args>
bool launch_pdl_cluster(void (*kernel)(KArgs...), unsigned grid, int threads, int smem, unsigned cluster,
                        cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess;
}

inline bool set_smem(const void *kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// 3D TMA map of a [B][N][H*32] bf16 tensor: boxes of 64 features x box_rows
// tokens, 128-byte swizzle.
bool make_bf16_map(CUtensorMap *m, const void *base, int B, int N, int H, int box_rows);
// 3D view of a [B][N][row_bytes] byte tensor (E4M3 codes): boxes of box_inner
// bytes x box_rows tokens, swizzle of 0, 64 or 128 bytes.
bool make_u8_map(CUtensorMap *m, const void *base, int B, int N, long long row_bytes, int box_inner, int box_rows,
                 int swizzle_bytes);

// A rank-dimensional TMA map of a bf16 tensor (dims innermost first, byte
// strides of dims 1.., box extents), no swizzle, zero fill out of range.
bool make_bf16_map_nd(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                      const cuuint64_t *strides, const cuuint32_t *box);

// Query side on the tensor cores (bf16, H % 4 == 0, no RoPE): its own split
// plan (one CTA per SM), dq and the split sums of [dS | dZ] from q, dout, the
// state S_eff (seff) and its packed operand [S|Z|0] (bop), which also gives S^T.
bool bwd_q_tc_available(const Plan &p);
void bwd_q_tc_plan(Plan &p);
int launch_bwd_q_tc(const void *q, const void *dout, void *dq, const float *seff, const void *bop, float *bpart,
                    const Plan &p, cudaStream_t s);
int read_and_clear_bwd_k_flag(unsigned *flag_out);
int read_and_clear_bwd_q_flag(unsigned *flag_out);
int read_and_clear_conv_flag(unsigned *flag_out);
int launch_bounded_wait_selftest(cudaStream_t s);

// Device flag raised by a bounded wait that gave up; read-and-clear.
int read_and_clear_device_flag(cudaStream_t s, unsigned *flag_out);

}  // namespace la
