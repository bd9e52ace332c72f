// k_ffma.cu -- CUDA-core (FFMA) reduce and apply kernels.
//
// The path for fp32 inputs and for bf16 shapes the tensor-core kernels do not
// take (H not a multiple of 4).  Same arithmetic as the tensor-core path:
// fp32 products and fp32 sums, phi = ReLU, numerator-only RoPE.
//
//   reduce:  partial[b][h][n][p] = sum over the split's tokens of
//            [ psi(k)^T v | phi(k) ]       (KV_n and z_n of one split)
//   apply:   out_t = psi(q_t) S_eff / (phi(q_t) . Z_eff + eps)
//
// ("KV product then accumulate" and "each block needs KVsum plus its own KV":
// "Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı", section
// "Sabit Bellekli KV önbelleğe alma mekanizması".)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.cuh"

namespace la {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Position of token j of the call along RoPE axis ax (0 frame, 1 row, 2 column).
__device__ __forceinline__ int rope_pos(const Plan &p, long long j, int ax) {
    const long long per_frame = (long long)p.Hg * p.Wg;
    if (ax == 0) return p.t_offset + (int)(j / per_frame);
    const long long r = j % per_frame;
    return ax == 1 ? (int)(r / p.Wg) : (int)(r % p.Wg);
}

// Rotate pair pr of token j: (x0, x1) -> (x0 c - x1 s, x0 s + x1 c).
__device__ __forceinline__ void rope_pair(const Plan &p, long long j, int pr, float &x0, float &x1) {
    const float ang = (float)rope_pos(p, j, p.axis[pr]) * p.theta[pr];
    float s, c;
    sincosf(ang, &s, &c);
    const float a = x0, b = x1;
    x0 = a * c - b * s;
    x1 = a * s + b * c;
}

constexpr int kRedThreads = 256;
constexpr int kRedRows = 64;

// One CTA per (b, h, block n, split sp).
template <typename T>
__global__ void __launch_bounds__(kRedThreads)
reduce_ffma_kernel(const T *__restrict__ k, const T *__restrict__ v, float *__restrict__ partials,
                   Plan p) {
    __shared__ float rk[kRedRows][kD + 1];   // psi(k) (rotated when RoPE)
    __shared__ float fk[kRedRows][kD + 1];   // phi(k)
    __shared__ float fv[kRedRows][kD + 1];   // v

    long long id = blockIdx.x;
    const int sp = (int)(id % p.P); id /= p.P;
    const int n = (int)(id % p.nb); id /= p.nb;
    const int h = (int)(id % p.H); id /= p.H;
    const int b = (int)id;

    const long long blk0 = (long long)n * p.L;
    long long blk1 = blk0 + p.L;
    if (blk1 > p.N) blk1 = p.N;
    const long long t0 = blk0 + (long long)sp * p.chunk;
    long long t1 = t0 + p.chunk;
    if (t1 > blk1) t1 = blk1;

    float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    const int tid = threadIdx.x;
    const size_t row_stride = (size_t)p.H * kD;

    for (long long r0 = t0; r0 < t1; r0 += kRedRows) {
        // stage 64 token rows: each thread handles 4 feature pairs
        for (int w = tid; w < kRedRows * (kD / 2); w += kRedThreads) {
            const int r = w / (kD / 2), pr = w % (kD / 2);
            const long long t = r0 + r;
            float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
            if (t < t1) {
                const size_t off = ((size_t)b * p.N + t) * row_stride + (size_t)h * kD + 2 * pr;
                k0 = fmaxf(to_f(k[off]), 0.f);
                k1 = fmaxf(to_f(k[off + 1]), 0.f);
                v0 = to_f(v[off]);
                v1 = to_f(v[off + 1]);
            }
            fk[r][2 * pr] = k0;
            fk[r][2 * pr + 1] = k1;
            if (p.rope && t < t1) rope_pair(p, t, pr, k0, k1);
            rk[r][2 * pr] = k0;
            rk[r][2 * pr + 1] = k1;
            fv[r][2 * pr] = v0;
            fv[r][2 * pr + 1] = v1;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < kRedRows; ++r) {
#pragma unroll
            for (int q = 0; q < 5; ++q) {
                const int e = tid + q * kRedThreads;
                if (e < kD * kD) acc[q] = fmaf(rk[r][e / kD], fv[r][e % kD], acc[q]);
                else if (e < kKVZ) acc[q] += fk[r][e - kD * kD];
            }
        }
        __syncthreads();
    }
    float *dst = partials + ((((size_t)b * p.H + h) * p.nb + n) * p.P + sp) * kKVZ;
#pragma unroll
    for (int q = 0; q < 5; ++q) {
        const int e = tid + q * kRedThreads;
        if (e < kKVZ) dst[e] = acc[q];
    }
}

constexpr int kAppThreads = 128;

// One CTA per (b, block n, head h, tile of 128 tokens); one thread per token.
template <typename T>
__global__ void __launch_bounds__(kAppThreads)
apply_ffma_kernel(const T *__restrict__ q, T *__restrict__ out, const float *__restrict__ seff,
                  Plan p) {
    __shared__ float S[kKVZ];
    const int tiles = (p.L + kAppThreads - 1) / kAppThreads;
    long long id = blockIdx.x;
    const int tile = (int)(id % tiles); id /= tiles;
    const int h = (int)(id % p.H); id /= p.H;
    const int n = (int)(id % p.nb); id /= p.nb;
    const int b = (int)id;

    const float *src = seff + (((size_t)b * p.H + h) * p.nb + n) * kKVZ;
    for (int e = threadIdx.x; e < kKVZ; e += kAppThreads) S[e] = src[e];
    __syncthreads();

    const long long blk0 = (long long)n * p.L;
    long long blk1 = blk0 + p.L;
    if (blk1 > p.N) blk1 = p.N;
    const long long t = blk0 + (long long)tile * kAppThreads + threadIdx.x;
    if (t >= blk1) return;

    const size_t off = ((size_t)b * p.N + t) * (size_t)p.H * kD + (size_t)h * kD;
    float fq[kD], rq[kD];
#pragma unroll
    for (int e = 0; e < kD; ++e) fq[e] = fmaxf(to_f(q[off + e]), 0.f);
#pragma unroll
    for (int pr = 0; pr < kD / 2; ++pr) {
        float a = fq[2 * pr], c = fq[2 * pr + 1];
        if (p.rope) rope_pair(p, t, pr, a, c);
        rq[2 * pr] = a;
        rq[2 * pr + 1] = c;
    }
    float den = 0.f;
#pragma unroll
    for (int e = 0; e < kD; ++e) den = fmaf(fq[e], S[kD * kD + e], den);
    const float inv = 1.0f / (den + p.eps);
#pragma unroll 4
    for (int j = 0; j < kD; ++j) {
        float num = 0.f;
#pragma unroll
        for (int e = 0; e < kD; ++e) num = fmaf(rq[e], S[e * kD + j], num);
        store_out(out + off + j, num * inv);
    }
}

}  // namespace

int launch_reduce_ffma(int is_bf16, const void *k, const void *v, float *partials, const Plan &p,
                       cudaStream_t s) {
    const long long grid = (long long)p.B * p.H * p.nb * p.P;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    if (is_bf16)
        reduce_ffma_kernel<__nv_bfloat16><<<(unsigned)grid, kRedThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), partials, p);
    else
        reduce_ffma_kernel<float><<<(unsigned)grid, kRedThreads, 0, s>>>(
            static_cast<const float *>(k), static_cast<const float *>(v), partials, p);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_apply_ffma(int is_bf16, const void *q, void *out, const float *seff, const Plan &p,
                      cudaStream_t s) {
    const long long tiles = (p.L + kAppThreads - 1) / kAppThreads;
    const long long grid = (long long)p.B * p.nb * p.H * tiles;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    if (is_bf16)
        apply_ffma_kernel<__nv_bfloat16><<<(unsigned)grid, kAppThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(out), seff, p);
    else
        apply_ffma_kernel<float><<<(unsigned)grid, kAppThreads, 0, s>>>(
            static_cast<const float *>(q), static_cast<float *>(out), seff, p);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace la
