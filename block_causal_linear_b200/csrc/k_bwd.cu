// k_bwd.cu -- backward pass of block-causal linear attention (CUDA cores).
//
// The pages give the forward recurrence only ("Nvidia, MIT ve diğerleri video
// yapay zeka devrimini başlattı", section "Sabit Bellekli KV önbelleğe alma
// mekanizması": KV_n accumulated into one cumulative state, every token of
// block n reads KVsum + its own block's KV); training a block-autoregressive
// model needs its derivative.  With S_n, Z_n the inclusive prefix state after
// block n (from the forward reduce and combine), per (b, h) and token t of
// block n:
//   num_t = psi(q_t) S_n,  den_t = phi(q_t) . Z_n + eps,
//   g_t = dout_t / den_t,  c_t = -(dout_t . num_t) / den_t^2,
//   dq_t = 1[q_t > 0] (R^T (S_n g_t) + c_t Z_n)
//   [dS_n | dZ_n] = sum_t [psi(q_t) g_t^T | c_t phi(q_t)]     (bwd_q_kernel)
//   G_m = sum_{n >= m} [dS_n | dZ_n]  in fixed order             (bwd_finish_kernel)
//   dk_t = 1[k_t > 0] (R^T (G_m v_t) + Gz_m),  dv_t = G_m^T psi(k_t)   (bwd_k_kernel)
// fp32 arithmetic, fixed summation orders (no atomics): repeated runs give the
// same bits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.cuh"

namespace la {
namespace {

__device__ __forceinline__ float ldf(const float *p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float *p, float x) { *p = x; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Angle of feature pair pr of token j of the call (numerator RoPE).
__device__ __forceinline__ float pair_angle(const Plan &p, long long j, int pr) {
    const long long per_frame = (long long)p.Hg * p.Wg;
    const int ax = p.axis[pr];
    long long pos;
    if (ax == 0) pos = p.t_offset + j / per_frame;
    else if (ax == 1) pos = (j % per_frame) / p.Wg;
    else pos = (j % per_frame) % p.Wg;
    return (float)pos * p.theta[pr];
}

// (x0, x1) -> R(+/-angle) (x0, x1): sgn = +1 rotates (psi), -1 the transpose.
__device__ __forceinline__ void rot_pair(float ang, float sgn, float &x0, float &x1) {
    float s, c;
    sincosf(ang, &s, &c);
    s *= sgn;
    const float a = x0, b = x1;
    x0 = a * c - b * s;
    x1 = a * s + b * c;
}

constexpr int kBThreads = 256;
constexpr int kBRows = 64;       // token rows per staging round (4 threads per row)

// One CTA per (b, h, block n, split sp): dq of the split's tokens and the
// split's [dS | dZ] sums.  seff: [B][H][nb][1056] inclusive prefix state.
template <typename T>
__global__ void __launch_bounds__(kBThreads)
bwd_q_kernel(const T *__restrict__ q, const T *__restrict__ dout, const float *__restrict__ seff,
             T *__restrict__ dq, float *__restrict__ bpart, Plan p) {
    __shared__ float Ss[kKVZ];                 // S_n (row = key feature), then Z_n
    __shared__ float pq[kBRows][kD + 1];       // psi(q)
    __shared__ float fq[kBRows][kD + 1];       // phi(q)
    __shared__ float gg[kBRows][kD + 1];       // g = dout / den
    __shared__ float cc[kBRows];               // c = -(dout . num) / den^2

    long long id = blockIdx.x;
    const int sp = (int)(id % p.P); id /= p.P;
    const int n = (int)(id % p.nb); id /= p.nb;
    const int h = (int)(id % p.H); id /= p.H;
    const int b = (int)id;
    const long long blk0 = (long long)n * p.L;
    const long long blk1 = blk0 + p.L < p.N ? blk0 + p.L : (long long)p.N;
    const long long t0 = blk0 + (long long)sp * p.chunk;
    const long long t1 = t0 + p.chunk < blk1 ? t0 + p.chunk : blk1;
    const int tid = threadIdx.x;
    const size_t bh = (size_t)b * p.H + h;

    const float *src = seff + (bh * p.nb + n) * kKVZ;
    for (int e = tid; e < kKVZ; e += kBThreads) Ss[e] = src[e];
    float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    const int r4 = tid >> 2, part = tid & 3;   // row of the round, quarter of the features
    const size_t row_stride = (size_t)p.H * kD;
    __syncthreads();

    for (long long r0 = t0; r0 < t1; r0 += kBRows) {
        const long long t = r0 + r4;
        const bool valid = t < t1;
        const size_t off = ((size_t)b * p.N + (valid ? t : t0)) * row_stride + (size_t)h * kD;
        // this thread's 8 features: phi, psi, and its 8 of the 32 num, dout terms
        float f[8], ps[8], dd[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const float x = valid ? ldf(q + off + 8 * part + a) : 0.f;
            f[a] = fmaxf(x, 0.f);
            ps[a] = f[a];
            dd[a] = valid ? ldf(dout + off + 8 * part + a) : 0.f;
        }
        if (p.rope && valid)
#pragma unroll
            for (int a = 0; a < 8; a += 2) rot_pair(pair_angle(p, t, (8 * part + a) / 2), 1.f, ps[a], ps[a + 1]);
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            pq[r4][8 * part + a] = ps[a];
            fq[r4][8 * part + a] = f[a];
        }
        __syncwarp();
        // den = phi(q) . Z (4 threads of the row, fixed order), num_j for j in
        // this thread's quarter, dn = dout . num
        float den = 0.f;
#pragma unroll
        for (int a = 0; a < 8; ++a) den = fmaf(f[a], Ss[kD * kD + 8 * part + a], den);
        den += __shfl_xor_sync(0xffffffffu, den, 1);
        den += __shfl_xor_sync(0xffffffffu, den, 2);
        den += p.eps;
        float dn = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = 8 * part + j;
            float num = 0.f;
#pragma unroll 8
            for (int a = 0; a < kD; ++a) num = fmaf(pq[r4][a], Ss[a * kD + c], num);
            dn = fmaf(dd[j], num, dn);
        }
        dn += __shfl_xor_sync(0xffffffffu, dn, 1);
        dn += __shfl_xor_sync(0xffffffffu, dn, 2);
        const float inv = 1.0f / den;
        const float cr = valid ? -dn * inv * inv : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) gg[r4][8 * part + j] = valid ? dd[j] * inv : 0.f;
        if (part == 0) cc[r4] = cr;
        __syncwarp();
        // dq: R^T (S g) + c Z on this thread's 8 features, ReLU mask
        if (valid) {
            float dp[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                float s = 0.f;
#pragma unroll 8
                for (int c = 0; c < kD; ++c) s = fmaf(Ss[(8 * part + a) * kD + c], gg[r4][c], s);
                dp[a] = s;
            }
            if (p.rope)
#pragma unroll
                for (int a = 0; a < 8; a += 2) rot_pair(pair_angle(p, t, (8 * part + a) / 2), -1.f, dp[a], dp[a + 1]);
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const float g = fmaf(cr, Ss[kD * kD + 8 * part + a], dp[a]);
                stf(dq + off + 8 * part + a, f[a] > 0.f ? g : 0.f);
            }
        }
        __syncthreads();
        // [dS | dZ] += [psi(q) g^T | c phi(q)] over the round's rows, row order
        const int rows = t1 - r0 < kBRows ? (int)(t1 - r0) : kBRows;
        for (int r = 0; r < rows; ++r) {
#pragma unroll
            for (int u = 0; u < 5; ++u) {
                const int e = tid + u * kBThreads;
                if (e < kD * kD) acc[u] = fmaf(pq[r][e / kD], gg[r][e % kD], acc[u]);
                else if (e < kKVZ) acc[u] = fmaf(cc[r], fq[r][e - kD * kD], acc[u]);
            }
        }
        __syncthreads();
    }
    float *dst = bpart + ((bh * p.nb + n) * p.P + sp) * kKVZ;
#pragma unroll
    for (int u = 0; u < 5; ++u) {
        const int e = tid + u * kBThreads;
        if (e < kKVZ) dst[e] = acc[u];
    }
}

// One thread per (b, h, number e of [dS | dZ]): suffix sums over blocks, last
// block first, the P splits of a block in split order.
__global__ void __launch_bounds__(kBThreads)
bwd_finish_kernel(const float *__restrict__ bpart, float *__restrict__ G, Plan p) {
    const long long w = (long long)blockIdx.x * kBThreads + threadIdx.x;
    if (w >= (long long)p.B * p.H * kKVZ) return;
    const size_t bh = (size_t)(w / kKVZ);
    const int e = (int)(w % kKVZ);
    float run = 0.f;
    for (int n = p.nb - 1; n >= 0; --n) {
        const float *src = bpart + (bh * p.nb + n) * p.P * kKVZ + e;
        for (int s = 0; s < p.P; ++s) run += src[(size_t)s * kKVZ];
        G[(bh * p.nb + n) * kKVZ + e] = run;
    }
}

constexpr int kKThreads = 128;

// One CTA per (b, block m, head h, tile of 128 tokens); one thread per token.
template <typename T>
__global__ void __launch_bounds__(kKThreads)
bwd_k_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ G,
             T *__restrict__ dk, T *__restrict__ dv, Plan p) {
    __shared__ float Gs[kKVZ];
    const int tiles = (p.L + kKThreads - 1) / kKThreads;
    long long id = blockIdx.x;
    const int tile = (int)(id % tiles); id /= tiles;
    const int h = (int)(id % p.H); id /= p.H;
    const int m = (int)(id % p.nb); id /= p.nb;
    const int b = (int)id;
    const float *src = G + (((size_t)b * p.H + h) * p.nb + m) * kKVZ;
    for (int e = threadIdx.x; e < kKVZ; e += kKThreads) Gs[e] = src[e];
    __syncthreads();

    const long long blk0 = (long long)m * p.L;
    const long long blk1 = blk0 + p.L < p.N ? blk0 + p.L : (long long)p.N;
    const long long t = blk0 + (long long)tile * kKThreads + threadIdx.x;
    if (t >= blk1) return;
    const size_t off = ((size_t)b * p.N + t) * (size_t)p.H * kD + (size_t)h * kD;
    float f[kD], ps[kD], vv[kD];
#pragma unroll
    for (int a = 0; a < kD; ++a) {
        f[a] = fmaxf(ldf(k + off + a), 0.f);
        ps[a] = f[a];
        vv[a] = ldf(v + off + a);
    }
    if (p.rope)
#pragma unroll
        for (int a = 0; a < kD; a += 2) rot_pair(pair_angle(p, t, a / 2), 1.f, ps[a], ps[a + 1]);
    // dv_c = sum_a G[a][c] psi(k)_a
#pragma unroll 4
    for (int c = 0; c < kD; ++c) {
        float s = 0.f;
#pragma unroll
        for (int a = 0; a < kD; ++a) s = fmaf(Gs[a * kD + c], ps[a], s);
        stf(dv + off + c, s);
    }
    // d psi(k)_a = sum_c G[a][c] v_c, then R^T, + Gz, ReLU mask
    float dp[kD];
#pragma unroll
    for (int a = 0; a < kD; ++a) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < kD; ++c) s = fmaf(Gs[a * kD + c], vv[c], s);
        dp[a] = s;
    }
    if (p.rope)
#pragma unroll
        for (int a = 0; a < kD; a += 2) rot_pair(pair_angle(p, t, a / 2), -1.f, dp[a], dp[a + 1]);
#pragma unroll
    for (int a = 0; a < kD; ++a) stf(dk + off + a, f[a] > 0.f ? dp[a] + Gs[kD * kD + a] : 0.f);
}

}  // namespace

int launch_bwd_q(int is_bf16, const void *q, const void *dout, const float *seff, void *dq, float *bpart,
                 const Plan &p, cudaStream_t s) {
    const long long grid = (long long)p.B * p.H * p.nb * p.P;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    if (is_bf16)
        bwd_q_kernel<__nv_bfloat16><<<(unsigned)grid, kBThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(dout), seff,
            static_cast<__nv_bfloat16 *>(dq), bpart, p);
    else
        bwd_q_kernel<float><<<(unsigned)grid, kBThreads, 0, s>>>(static_cast<const float *>(q),
                                                                 static_cast<const float *>(dout), seff,
                                                                 static_cast<float *>(dq), bpart, p);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_bwd_finish(const float *bpart, float *G, const Plan &p, cudaStream_t s) {
    const long long threads = (long long)p.B * p.H * kKVZ;
    const long long grid = (threads + kBThreads - 1) / kBThreads;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    bwd_finish_kernel<<<(unsigned)grid, kBThreads, 0, s>>>(bpart, G, p);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_bwd_k(int is_bf16, const void *k, const void *v, const float *G, void *dk, void *dv, const Plan &p,
                 cudaStream_t s) {
    const long long tiles = (p.L + kKThreads - 1) / kKThreads;
    const long long grid = (long long)p.B * p.nb * p.H * tiles;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    if (is_bf16)
        bwd_k_kernel<__nv_bfloat16><<<(unsigned)grid, kKThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), G,
            static_cast<__nv_bfloat16 *>(dk), static_cast<__nv_bfloat16 *>(dv), p);
    else
        bwd_k_kernel<float><<<(unsigned)grid, kKThreads, 0, s>>>(static_cast<const float *>(k),
                                                                 static_cast<const float *>(v), G,
                                                                 static_cast<float *>(dk), static_cast<float *>(dv),
                                                                 p);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace la
