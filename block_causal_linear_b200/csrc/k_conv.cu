// k_conv.cu -- depthwise 3D convolution of the Spatial-Temporal Mix-FFN.
//
// "Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı", section
// "Verimli doğrusal DiT": the MLP alternates a 1x3x3 spatial and a 3x1x1
// temporal convolution to add local information to every token.  Depthwise
// (one filter per channel), zero padding inside the call's frames:
//   y[b,t,h,w,c] = bias[c] + sum_taps w[c][i][j][l] x[b, t+i-pt, h+j-ph, w+l-pw, c]
// x, y: [B][T][Hg][Wg][C], channels last (the token layout of the attention).
//
// HBM-bound stencil: each thread owns 8 channels (one 16-byte bf16 vector, two
// fp32 vectors) with their taps and bias in registers and walks a run of
// consecutive tokens; a warp reads 32 consecutive channel vectors of a token
// per tap (coalesced), and the neighbour tokens a tap reaches (one row or one
// frame away) are read again by CTAs running at the same time, from L2.  fp32
// accumulation in a fixed tap order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kCThreads = 256;
constexpr int kCTokens = 32;     // tokens per CTA run

__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void store8(float *p, const float (&v)[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ uint32_t bf2c(float a, float b) {
    const __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&t);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&v)[8]) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(bf2c(v[0], v[1]), bf2c(v[2], v[3]), bf2c(v[4], v[5]), bf2c(v[6], v[7]));
}

// grid: x = runs of kCTokens tokens, y = blocks of kCThreads channel vectors.
template <typename T, int KT, int KH, int KW>
__global__ void __launch_bounds__(kCThreads)
dwconv_kernel(const T *__restrict__ x, T *__restrict__ y, const float *__restrict__ wgt,
              const float *__restrict__ bias, int B, int Tf, int Hg, int Wg, int C) {
    constexpr int kTaps = KT * KH * KW;
    const int cv = blockIdx.y * kCThreads + threadIdx.x;   // channel vector: channels 8cv .. 8cv+7
    if (8 * cv >= C) return;
    float wr[kTaps][8], acc0[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int c = 8 * cv + k;
        acc0[k] = bias ? bias[c] : 0.f;
#pragma unroll
        for (int tp = 0; tp < kTaps; ++tp) wr[tp][k] = wgt[(size_t)c * kTaps + tp];
    }
    const long long ntok = (long long)B * Tf * Hg * Wg;
    long long tok = (long long)blockIdx.x * kCTokens;
    if (tok >= ntok) return;
    // position of the run's first token, then stepped token by token
    long long r = tok;
    int w0 = (int)(r % Wg); r /= Wg;
    int h0 = (int)(r % Hg); r /= Hg;
    int t0 = (int)(r % Tf);
    const int tend = (int)((ntok - tok) < kCTokens ? (ntok - tok) : kCTokens);
    for (int i = 0; i < tend; ++i, ++tok) {
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = acc0[k];
#pragma unroll
        for (int a = 0; a < KT; ++a) {
            const int dt = a - KT / 2;
            if (t0 + dt < 0 || t0 + dt >= Tf) continue;
#pragma unroll
            for (int bq = 0; bq < KH; ++bq) {
                const int dh = bq - KH / 2;
                if (h0 + dh < 0 || h0 + dh >= Hg) continue;
#pragma unroll
                for (int l = 0; l < KW; ++l) {
                    const int dw = l - KW / 2;
                    if (w0 + dw < 0 || w0 + dw >= Wg) continue;
                    const long long src = tok + ((long long)dt * Hg + dh) * Wg + dw;
                    float v[8];
                    load8(x + src * C + 8 * cv, v);
                    const int tp = (a * KH + bq) * KW + l;
#pragma unroll
                    for (int k = 0; k < 8; ++k) acc[k] = fmaf(wr[tp][k], v[k], acc[k]);
                }
            }
        }
        store8(y + tok * C + 8 * cv, acc);
        if (++w0 == Wg) {
            w0 = 0;
            if (++h0 == Hg) {
                h0 = 0;
                if (++t0 == Tf) t0 = 0;
            }
        }
    }
}

template <int KT, int KH, int KW>
int launch_shape(int is_bf16, const void *x, void *y, const float *w, const float *bias, int B, int T, int Hg,
                 int Wg, int C, cudaStream_t s) {
    const long long ntok = (long long)B * T * Hg * Wg;
    const long long gx = (ntok + kCTokens - 1) / kCTokens;
    const long long gy = ((long long)C / 8 + kCThreads - 1) / kCThreads;
    if (gx <= 0 || gx > 0x7fffffffLL || gy > 65535) return -1;
    const dim3 grid((unsigned)gx, (unsigned)gy);
    if (is_bf16)
        dwconv_kernel<__nv_bfloat16, KT, KH, KW><<<grid, kCThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(y), w, bias, B, T, Hg, Wg, C);
    else
        dwconv_kernel<float, KT, KH, KW><<<grid, kCThreads, 0, s>>>(static_cast<const float *>(x),
                                                                    static_cast<float *>(y), w, bias, B, T, Hg, Wg,
                                                                    C);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

int launch_dwconv(int is_bf16, const void *x, void *y, const float *w, const float *bias, int B, int T, int Hg,
                  int Wg, int C, int kt, int kh, int kw, cudaStream_t s) {
    if (kt == 1 && kh == 3 && kw == 3) return launch_shape<1, 3, 3>(is_bf16, x, y, w, bias, B, T, Hg, Wg, C, s);
    if (kt == 3 && kh == 1 && kw == 1) return launch_shape<3, 1, 1>(is_bf16, x, y, w, bias, B, T, Hg, Wg, C, s);
    return -2;   // not a Mix-FFN kernel shape
}

}  // namespace la
