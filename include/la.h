/*
 * la.h -- C ABI of libla_b200.so: block-causal linear attention with a
 * constant-memory fp32 state, on NVIDIA B200 (sm_100a).
 *
 * The operation (sources cited by page title and section):
 *   - "Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı"
 *     (aihaber.org), section "Sabit Bellekli KV önbelleğe alma mekanizması":
 *     a video is cut into blocks; later blocks see earlier ones through linear
 *     attention, never the reverse; the KV products of the blocks are summed
 *     (KV_{1-2} = KV_1 + KV_2, ...) into a cache of fixed size; each block
 *     needs only that sum plus its own KV.
 *   - sd114.wiki SANA-Video summary, section "两大核心技术突破": item 1, linear
 *     attention as a kernel feature map plus global aggregation, with RoPE for
 *     spatio-temporal position; item 2, chunk-wise linear attention whose only
 *     context is one cumulative state, constant in memory.
 *   - "SANA-Video: Efficient Video Generation with Block Linear Diffusion
 *     Transformer" (chatpaper.ai abstract), design (2): the constant-memory
 *     state replaces a growing KV cache.
 *
 * Per batch element b and head h, with phi = ReLU applied elementwise:
 *   KV_n = sum_{t in block n} psi(k_t)^T v_t      (d x d, fp32)
 *   z_n  = sum_{t in block n} phi(k_t)            (d, fp32)
 *   out_t = psi(q_t) (S + KV_n) / ( phi(q_t) . (Z + z_n) + eps )   for t in block n
 * where S, Z are the sums over earlier blocks.  psi = phi, or with RoPE
 * psi = R(position) o phi in the numerator only.
 *
 * Conventions for every entry point
 *   - Tensors q, k, v, out are DEVICE pointers, row-major [B][N][H][d] with d
 *     fastest, element type given by la_dtype (out has the input type; bf16 out
 *     is rounded to nearest even from fp32).  Base addresses must be 16-byte
 *     aligned.  d must be 32.
 *   - The caller owns every buffer (q, k, v, out, S, Z, workspace) and keeps it
 *     alive until the enqueued work has finished.  The library allocates no
 *     device memory and never synchronises; all work is enqueued on `stream`
 *     (a cudaStream_t passed as void*, NULL = legacy default stream).
 *   - Validation is synchronous and happens before anything is enqueued; an
 *     error status means nothing was enqueued.  No C++ exception crosses the ABI.
 *   - Results are deterministic: identical inputs and shapes on the same GPU
 *     model give bitwise-identical out, S and Z (fixed reduction order, no
 *     floating-point atomics).
 *   - Inputs must be finite.
 */
#ifndef LA_B200_LA_H
#define LA_B200_LA_H

#include <stddef.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_EINVAL = 1,        /* null pointer, bad size, misaligned pointer, bad RoPE */
    LA_EUNSUPPORTED = 2,  /* d != 32, or a shape this build does not handle */
    LA_ECUDA = 3,         /* a CUDA call or kernel launch failed */
    LA_ETIMEOUT = 4,      /* a device-side bounded wait gave up (la_device_status) */
    LA_EWORKSPACE = 5     /* workspace null or smaller than la_workspace_size() */
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

/*
 * 3D rotary position embedding (RoPE) on phi(q), phi(k) in the numerator.
 * The d features are cut into sections of dt, dh, dw dims (each even, sum d)
 * for the latent frame, row and column.  Inside a section of D dims, features
 * (2i, 2i+1) rotate by angle pos * base^(-2i/D):
 *   x'_{2i} = x_{2i} cos - x_{2i+1} sin,   x'_{2i+1} = x_{2i} sin + x_{2i+1} cos.
 * Token j of a call (0-based, in token order) sits at frame t_offset + j/(Hg*Wg),
 * row (j % (Hg*Wg)) / Wg, column j % Wg.  The pages name RoPE but fix neither
 * pairing, sections nor frequencies; this is the library's stated reading.
 */
typedef struct {
    int T;          /* latent frames per block: la_block_forward with commit advances
                       state->t_next by T */
    int Hg, Wg;     /* latent rows and columns per frame, > 0 */
    int t_offset;   /* frame of token 0 of the call; < 0 in la_block_forward means
                       "use state->t_next" */
    int dt, dh, dw; /* section dims, even, dt + dh + dw == d */
    float base;     /* frequency base, > 0 (10000 in SANA-style 3D RoPE) */
} la_rope;

/*
 * The constant-memory state of the streaming method: per (b, h) the running
 * S = sum KV_i (d x d) and Z = sum z_i (d) over committed blocks, fp32.
 * S and Z are caller-owned DEVICE buffers of B*H*d*d and B*H*d floats,
 * layout S[b][h][row = key feature][column = value feature], Z[b][h][feature].
 * Their size never depends on how many blocks have been committed.
 * blocks_committed and t_next are host-side counters kept by the library.
 * Saving and restoring S, Z and the two counters checkpoints the stream.
 */
typedef struct {
    float *S;
    float *Z;
    int B, H, d;
    long long blocks_committed;
    int t_next;
} la_state;

/*
 * Bytes of caller-provided device workspace that la_full_forward needs for
 * these sizes (tokens_per_block 0 = one block of N tokens), and that
 * la_block_forward needs with N = tokens_per_block = N_blk.  Pure host
 * function, no CUDA call.  Returns 0 for invalid sizes.  The workspace holds
 * the split partial sums, the per-block effective state and the packed
 * tensor-core operand; its size never depends on how many blocks were
 * streamed before.  Its base must be 256-byte aligned.
 * The pages have no counterpart of this call: they describe the block sum
 * KV_n as one reduction ("Nvidia, MIT ve diğerleri video yapay zeka
 * devrimini başlattı", section "Sabit Bellekli KV önbelleğe alma
 * mekanizması"); the workspace is where this library keeps the pieces of
 * that reduction when it cuts a block's tokens into splits to fill the GPU.
 */
LA_API size_t la_workspace_size(int B, int N, int H, int d, int tokens_per_block);

/*
 * Start a stream: bind the caller's S, Z buffers to *st, zero them
 * (cudaMemsetAsync on `stream`) and reset blocks_committed and t_next to 0.
 * Source: "Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı"
 * (aihaber.org), section "Sabit Bellekli KV önbelleğe alma mekanizması": the
 * cache is empty before block 1 and receives block 1's KV first; sd114.wiki
 * SANA-Video summary, section "两大核心技术突破", item 2: the only context a
 * chunk sees is one cumulative state of constant size.  Zero S, Z is that
 * empty cache, so block 1 sees only itself.
 * Errors: null st, S or Z, or S, Z not 16-byte aligned, or B, H <= 0:
 * LA_EINVAL; d != 32: LA_EUNSUPPORTED; a failed memset: LA_ECUDA.
 */
LA_API la_status la_state_init(la_state *st, float *S, float *Z, int B, int H, int d, void *stream);

/*
 * Checkpoint and resume of a stream.  All the method keeps of the past is the
 * fixed-size state ("Nvidia, MIT ve diğerleri video yapay zeka devrimini
 * başlattı", section "Sabit Bellekli KV önbelleğe alma mekanizması": the cache
 * holds only the running sum of the blocks' KV; sd114.wiki, section
 * "两大核心技术突破", item 2: one cumulative state of constant size), so S, Z
 * and the two host counters are a complete checkpoint of any stream.
 * la_state_save: copies st's S and Z to S_dst (B*H*d*d floats) and Z_dst
 *   (B*H*d floats), host or device memory, with one cudaMemcpyAsync each
 *   (cudaMemcpyDefault) on `stream`, and stores the counters in *counters at
 *   once.  The copies are complete when `stream` reaches them (pinned host
 *   memory keeps them asynchronous).
 * la_state_restore: copies S_src, Z_src into st's S, Z the same way and sets
 *   st's counters from *counters.  st must be bound by la_state_init with the
 *   checkpoint's B, H, d.
 * Streaming blocks after a restore gives bitwise the results of streaming on
 * from the saved point.  Errors: a null or unbound st, a null buffer or
 * counters pointer, or negative counters: LA_EINVAL; a failed copy: LA_ECUDA.
 */
typedef struct {
    long long blocks_committed;
    int t_next;
} la_state_counters;
LA_API la_status la_state_save(const la_state *st, float *S_dst, float *Z_dst, la_state_counters *counters,
                               void *stream);
LA_API la_status la_state_restore(la_state *st, const float *S_src, const float *Z_src,
                                  const la_state_counters *counters, void *stream);

/*
 * One block of the streaming method.  Source: "Nvidia, MIT ve diğerleri video
 * yapay zeka devrimini başlattı" (aihaber.org), section "Sabit Bellekli KV
 * önbelleğe alma mekanizması": a block needs only the cached sum of the
 * earlier blocks' KV plus its own KV, and its KV is then added to the cache;
 * later blocks never reach back into earlier tokens.  For the N_blk tokens of
 * this block:
 *   S_eff = S + KV_n,  Z_eff = Z + z_n,  out = psi(q) S_eff / (phi(q).Z_eff + eps),
 * every token of the block attending to every other token of it
 * (bidirectional inside the block) and to all committed blocks.
 * commit != 0: S <- S_eff, Z <- Z_eff on the device, blocks_committed += 1,
 *   t_next += rope ? rope->T : 0.
 * commit == 0: a read-only pass (e.g. a denoising step before the last); S, Z
 *   stay bitwise unchanged.
 * rope may be NULL.  st must have been set up by la_state_init with the same
 * B, H, d.  ws must hold la_workspace_size(B, N_blk, H, d, N_blk) bytes.
 * The host counters advance when the call is enqueued.  If a later
 * la_device_status reports LA_ETIMEOUT, a committing call enqueued since the
 * last successful la_device_status may have left S, Z partly updated while
 * the counters say it committed: restore the last checkpoint
 * (la_state_restore) or start over with la_state_init before streaming on.
 * Errors: as la_full_forward, plus LA_EINVAL for a null or unbound st or one
 * of other shapes.
 */
LA_API la_status la_block_forward(const void *q, const void *k, const void *v, void *out, la_dtype dt,
                           int B, int N_blk, int H, int d, la_state *st, int commit,
                           const la_rope *rope, float eps, void *ws, size_t ws_bytes,
                           void *stream);

/*
 * The whole sequence from a zero state in one call.  Source: "Nvidia, MIT ve
 * diğerleri video yapay zeka devrimini başlattı" (aihaber.org), section
 * "Sabit Bellekli KV önbelleğe alma mekanizması": block 1's KV is cached,
 * block 2 adds its KV to the cache (KV_{1-2} = KV_1 + KV_2), and so on until
 * the last block's sum is the KV of the whole video; every block sees the
 * cached sum plus its own KV.  Blocks of tokens_per_block tokens (0 = a
 * single bidirectional block of all N tokens; the last block may be
 * shorter), block n seeing blocks 0..n.  Equal to la_state_init followed by
 * la_block_forward(commit=1) on each block, up to the order of fp32 sums.
 * rope may be NULL; positions run over the whole sequence (t_offset >= 0).
 * ws must hold la_workspace_size(B, N, H, d, tokens_per_block) bytes.
 * Errors: null or not 16-byte aligned q, k, v, out, a bad dtype, size, eps
 * or RoPE: LA_EINVAL; d != 32: LA_EUNSUPPORTED; ws null, too small or not
 * 256-byte aligned: LA_EWORKSPACE; a failed launch: LA_ECUDA.
 */
LA_API la_status la_full_forward(const void *q, const void *k, const void *v, void *out, la_dtype dt,
                          int B, int N, int H, int d, int tokens_per_block,
                          const la_rope *rope, float eps, void *ws, size_t ws_bytes,
                          void *stream);

/*
 * Backward pass of la_full_forward, for block-autoregressive training.  The
 * pages give the forward recurrence ("Nvidia, MIT ve diğerleri video yapay
 * zeka devrimini başlattı", section "Sabit Bellekli KV önbelleğe alma
 * mekanizması"); this is its derivative.  Given dout = d loss / d out for
 * la_full_forward(q, k, v, tokens_per_block, rope, eps) (zero initial state),
 * writes dq, dk, dv = d loss / d q, k, v:
 *   per (b, h), token t of block n, S_n and Z_n the state after block n:
 *   g_t = dout_t / den_t,  c_t = -(dout_t . num_t) / den_t^2,
 *   dq_t = 1[q_t > 0] (R^T (S_n g_t) + c_t Z_n),
 *   G_m = sum_{n >= m} sum_{t in n} [psi(q_t) g_t^T | c_t phi(q_t)],
 *   dk_t = 1[k_t > 0] (R^T (G_m v_t) + Gz_m),  dv_t = G_m^T psi(k_t)
 * (ReLU derivative 1[x > 0]; R the numerator rotation when rope is given).
 * Tensors: q, k, v, dout, dq, dk, dv all [B][N][H][d] of type dt, device
 * pointers, 16-byte aligned, caller-owned; dq, dk, dv may not overlap the
 * inputs.  ws must hold la_backward_workspace_size(B, N, H, d,
 * tokens_per_block) bytes (256-byte aligned), else LA_EWORKSPACE; argument
 * errors return LA_EINVAL / LA_EUNSUPPORTED before anything is enqueued.
 * fp32 sums in fixed orders: repeated calls give the same bits.
 */
LA_API size_t la_backward_workspace_size(int B, int N, int H, int d, int tokens_per_block);
LA_API la_status la_full_backward(const void *q, const void *k, const void *v, const void *dout,
                                  void *dq, void *dk, void *dv, la_dtype dt, int B, int N, int H,
                                  int d, int tokens_per_block, const la_rope *rope, float eps,
                                  void *ws, size_t ws_bytes, void *stream);

/*
 * FP8 inputs.  q, k, v as FP8 E4M3 codes (one byte each, [B][N][H][d], OCP
 * 8-bit float E4M3: bias 7, 3 mantissa bits, max 448) with one fp32 scale per
 * tensor: the values are q = scale_q * decode(q_code), and likewise k, v.
 * Since ReLU commutes with a positive scale, the results are those of
 * la_full_forward / la_block_forward on the decoded values:
 *   KV_n = scale_k scale_v sum phi(k^) v^T,  z_n = scale_k sum phi(k^),
 *   out = scale_q psi(q^) S_eff / (scale_q phi(q^) . Z_eff + eps),
 * out in bf16.  The state (S, Z) is fp32 in real units, so e4m3 and bf16
 * calls may share one stream of blocks.  The pages quantise the deployed
 * model to NVFP4 ("Nvidia, MIT ve diğerleri video yapay zeka devrimini
 * başlattı", section "Etkin eğitim ve çıkarım stratejileri": SVDQuant); FP8
 * q, k, v here shrink the bytes this path moves (160 instead of 256 per token
 * and head).
 * With rope, the rotation acts on phi(q^), phi(k^) as in the bf16 calls (a
 * rotation is linear, so the scales still factor out), and rope follows the
 * bf16 calls' rules (la_block_forward_e4m3: t_offset < 0 takes the state's
 * t_next, a commit advances it by rope->T).
 * Scales must be finite and > 0 (LA_EINVAL); H must be a multiple of 4 and
 * the GPU must take the tensor-core path, which with rope also needs the
 * call's cos/sin records (8 groups of 4 features, each group on one axis,
 * over the call's frames, rows and columns) to fit 8 KiB (else
 * LA_EUNSUPPORTED).  Workspace and every other argument as in the bf16 calls.
 */
LA_API la_status la_full_forward_e4m3(const void *q, const void *k, const void *v, float scale_q,
                                      float scale_k, float scale_v, void *out, int B, int N, int H,
                                      int d, int tokens_per_block, const la_rope *rope, float eps,
                                      void *ws, size_t ws_bytes, void *stream);
LA_API la_status la_block_forward_e4m3(const void *q, const void *k, const void *v, float scale_q,
                                       float scale_k, float scale_v, void *out, int B, int N_blk,
                                       int H, int d, la_state *st, int commit, const la_rope *rope,
                                       float eps, void *ws, size_t ws_bytes, void *stream);

/*
 * NVFP4 inputs, the format the pages deploy the model in ("Nvidia, MIT ve
 * diğerleri video yapay zeka devrimini başlattı", section "Etkin eğitim ve
 * çıkarım stratejileri": SVDQuant NVFP4).  Each of q, k, v is three parts:
 *   codes:       DEVICE uint8 [B][N][H][d/2], two FP4 E2M1 codes per byte
 *                (element 2i in the low nibble, 2i+1 in the high nibble;
 *                E2M1: sign, 2 exponent bits with bias 1, 1 mantissa bit,
 *                magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6);
 *   block scale: DEVICE uint8 [B][N][H][d/16], one FP8 E4M3 scale per 16
 *                consecutive features, sign bit clear (not NaN);
 *   scale_x:     one fp32 per-tensor scale, finite and > 0;
 * value = e2m1(code) * e4m3(block scale) * scale_x.  A positive scale
 * commutes with ReLU, so the results are those of la_full_forward /
 * la_block_forward on the decoded values (out = scale_q psi(q^) S_eff /
 * (scale_q phi(q^) . Z_eff + eps), KV and z carry scale_k scale_v and
 * scale_k), out in bf16, the state fp32 in real units.  q, k, v move 18
 * bytes per token and head each instead of 64.
 * With rope, the rotation acts on the decoded phi(q^), phi(k^) and rope
 * follows the bf16 calls' rules, as for the E4M3 calls.
 * Errors: null or not 16-byte aligned pointers, or a scale_x not finite and
 * > 0, LA_EINVAL; H not a multiple of 8, no tensor-core path, or a RoPE grid
 * whose cos/sin records do not fit 8 KiB, LA_EUNSUPPORTED.  A block scale
 * with the sign bit set or NaN gives unspecified values (no fault).
 * Workspace and every other argument as in the bf16 calls.
 */
LA_API la_status la_full_forward_nvfp4(const void *q, const void *k, const void *v,
                                       const void *q_blk_scale, const void *k_blk_scale,
                                       const void *v_blk_scale, float scale_q, float scale_k,
                                       float scale_v, void *out, int B, int N, int H, int d,
                                       int tokens_per_block, const la_rope *rope, float eps, void *ws,
                                       size_t ws_bytes, void *stream);
LA_API la_status la_block_forward_nvfp4(const void *q, const void *k, const void *v,
                                        const void *q_blk_scale, const void *k_blk_scale,
                                        const void *v_blk_scale, float scale_q, float scale_k,
                                        float scale_v, void *out, int B, int N_blk, int H, int d,
                                        la_state *st, int commit, const la_rope *rope, float eps,
                                        void *ws, size_t ws_bytes, void *stream);

/*
 * Depthwise 3D convolution of the Spatial-Temporal Mix-FFN, the step after
 * attention in a block ("Nvidia, MIT ve diğerleri video yapay zeka devrimini
 * başlattı", section "Verimli doğrusal DiT": the MLP alternates a 1x3x3
 * spatial and a 3x1x1 temporal convolution).  Reading: depthwise (one filter
 * per channel), zero padding of one at the edges of the call's frames, rows
 * and columns (a temporal tap never reaches another call's frames):
 *   y[b,t,h,w,c] = bias[c] + sum_{i,j,l} weight[c][i][j][l] x[b, t+i-pt, h+j-ph, w+l-pw, c]
 * x, y: DEVICE tensors [B][T][Hg][Wg][C] of type dt (channels last: the token
 * layout of q, k, v), 16-byte aligned, caller-owned, not overlapping.
 * weight: DEVICE fp32 [C][kt][kh][kw]; bias: DEVICE fp32 [C] or NULL.
 * (kt, kh, kw) must be (1, 3, 3) or (3, 1, 1) and C a multiple of 8, else
 * LA_EUNSUPPORTED; other argument errors LA_EINVAL.  fp32 accumulation.
 */
LA_API la_status la_dwconv3d(const void *x, void *y, la_dtype dt, int B, int T, int Hg, int Wg, int C,
                             int kt, int kh, int kw, const float *weight, const float *bias,
                             void *stream);

/*
 * Token split of one block over R GPUs (one process per GPU), for blocks
 * whose (batch, head) pairs are too few to fill the GPUs: rank r holds a
 * contiguous slice of the block's tokens (q, k, v [B][N_slice][H][d]).  The
 * block's KV_n and z_n are sums over its tokens ("Nvidia, MIT ve diğerleri
 * video yapay zeka devrimini başlattı", section "Sabit Bellekli KV önbelleğe
 * alma mekanizması"), so each rank reduces its slice, the ranks exchange the
 * B*H*(d*d + d) fp32 partial sums (an all-gather, the caller's collective,
 * e.g. NCCL), and each rank adds them to the state in rank order and applies
 * its own queries:
 *   la_block_reduce: partial[b][h] = [sum_{t in slice} psi(k_t)^T v_t | sum phi(k_t)]
 *     (fp32 DEVICE buffer of la_split_partial_bytes(B, H, d) bytes, layout of
 *     one [S | Z] per (b, h): 1024 + 32 floats);
 *   la_block_apply: gathered = the R ranks' partials, [R][B][H][d*d + d] in
 *     rank order (DEVICE, caller-owned); S_eff = S + partial_0 + ... +
 *     partial_{R-1} (that order), out for this rank's tokens, and on commit
 *     S <- S_eff on every rank alike (identical bits on all ranks).
 * With RoPE every slice must start at a frame boundary, rope->t_offset being
 * the frame of the slice's first token (la_block_apply: < 0 means the state's
 * t_next, which on commit advances by rope->T, the block's frames).  ws as
 * la_workspace_size(B, N_slice, H, d, N_slice).  R in [1, 32].  Errors as in
 * la_block_forward.
 */
LA_API size_t la_split_partial_bytes(int B, int H, int d);
LA_API la_status la_block_reduce(const void *k, const void *v, la_dtype dt, int B, int N_slice, int H,
                                 int d, const la_rope *rope, float *partial, void *ws,
                                 size_t ws_bytes, void *stream);
LA_API la_status la_block_apply(const void *q, void *out, la_dtype dt, int B, int N_slice, int H, int d,
                                const float *gathered, int R, la_state *st, int commit,
                                const la_rope *rope, float eps, void *ws, size_t ws_bytes,
                                void *stream);

/*
 * For callers that cannot allocate device memory at all.  Some code that
 * calls this library runs inside a host framework that owns every device
 * allocation and gives a plug-in no allocator and no way to size or keep a
 * workspace between calls (a video pipeline or inference-server plug-in on a
 * fixed memory budget, for example).  This variant of la_full_forward needs
 * no workspace argument: its scratch (the split partial sums, the effective
 * state and the packed tensor-core operand) lives in a static device array of
 * LA_STATIC_WS_BYTES bytes that the library defines at file scope.  Every GPU
 * that loads the library holds that array until the process exits.  The
 * pages have no counterpart of this entry point.
 *
 * Arguments and results are those of la_full_forward without ws/ws_bytes.
 * Shapes whose la_workspace_size() exceeds LA_STATIC_WS_BYTES are rejected
 * with LA_EWORKSPACE before anything is enqueued.  The call allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library routine).  The first call
 * on each device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream capture.
 * All calls on a device share the one array and it keeps the last call's
 * contents; each call writes every scratch byte it reads, so nothing needs to
 * start at zero, but calls whose work overlaps on the GPU (different streams,
 * no ordering between them) race on the array and give wrong results.
 */
#define LA_STATIC_WS_BYTES (16u << 20)
LA_API la_status la_full_forward_static_ws(const void *q, const void *k, const void *v, void *out,
                                           la_dtype dt, int B, int N, int H, int d,
                                           int tokens_per_block, const la_rope *rope, float eps,
                                           void *stream);

/*
 * Device-side status of the kernels enqueued so far on this device: every
 * wait inside a kernel is bounded; one that gives up records the fact in a
 * device flag and the kernel returns early.  This call synchronises `stream`,
 * reads and clears the flag, and returns LA_ETIMEOUT if it was set, LA_ECUDA
 * on a CUDA error, else LA_OK.  After LA_ETIMEOUT the outputs of the calls
 * enqueued since the last LA_OK are not valid, and a stream with committing
 * calls among them must be restored from a checkpoint (la_state_restore) or
 * restarted (la_state_init): their host counters advanced when they were
 * enqueued.
 */
LA_API la_status la_device_status(void *stream);

/*
 * Self-test of the bounded waits: enqueues on `stream` one small kernel whose
 * wait on a barrier that nothing arrives at gives up after the waits' time
 * limit (2 s) and raises the device flag, as a kernel's wait would after a
 * lost copy or a stalled partner.  The following la_device_status returns
 * LA_ETIMEOUT (and clears the flag).  No fault, no trap, the context stays
 * usable.  Returns LA_ECUDA if the launch failed, else LA_OK.
 */
LA_API la_status la_selftest_bounded_wait(void *stream);

/* Static, human-readable name of a status (never NULL; "unknown status" for
 * a value outside la_status).  The pages have no counterpart: it belongs to
 * the library's error reporting. */
LA_API const char *la_status_string(la_status s);

/*
 * Measurement hook.  When set (non-NULL cudaEvent_t handles passed as void*,
 * created on the current device), every following forward call records
 * before_reduce before its first kernel, after_reduce after the state
 * reduction, after_finish after the state combine and after_apply after its
 * last kernel, all on its stream (when the reduction combines its own splits,
 * after_reduce and after_finish are recorded back to back).  la_full_backward
 * records the same four events before its first kernel, after the forward
 * state (reduction and combine), after the query side (dq and the
 * state-gradient sums) and after the key side (suffix sums, dk, dv).  Pass
 * four NULLs to stop.
 * Process-global; not thread-safe.  Changes no result.
 */
LA_API void la_set_stage_events(void *before_reduce, void *after_reduce, void *after_finish,
                                void *after_apply);

/* Number of kernels the last successful forward call enqueued (for launch
 * accounting), and a short name of the path it took ("tc" or "ffma"). */
LA_API int la_last_launch_count(void);
/* 1 if this build routes bf16 inputs with H % 4 == 0 through the tensor-core
 * (tcgen05) kernels, 0 if every shape takes the CUDA-core kernels. */
LA_API int la_tc_enabled(void);
LA_API const char *la_last_path(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_B200_LA_H */
