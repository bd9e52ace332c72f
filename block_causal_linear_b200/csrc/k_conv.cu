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
// fp32 vectors) with their taps and bias in registers and slides a window of
// input vectors along the axis the taps repeat on (columns for 1x3x3, frames
// for 3x1x1), so an output costs 3 (spatial) or 1 (temporal) new loads; a warp
// reads 32 consecutive channel vectors of a token (coalesced); the rows above
// and below come again from L2, read by the CTAs of the neighbouring rows.
// fp32 accumulation in a fixed tap order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kCThreads = 128;   // 8-channel vectors per CTA

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

__device__ __forceinline__ void zero8(float (&v)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = 0.f;
}

// 1x3x3: one CTA per (b, t, h) row and block of kCThreads channel vectors;
// each thread slides a 3x3 window of 8-channel vectors (rows h-1, h, h+1)
// along the row, so an output needs the 3 vectors of one new column.
template <typename T>
__global__ void __launch_bounds__(kCThreads)
dwconv_spatial_kernel(const T *__restrict__ x, T *__restrict__ y, const float *__restrict__ wgt,
                      const float *__restrict__ bias, long long nrows, int Hg, int Wg, int C) {
    const int cv = blockIdx.x * kCThreads + threadIdx.x;   // channels 8cv .. 8cv+7
    if (8 * cv >= C) return;
    const long long row = (long long)blockIdx.z * 65535 + blockIdx.y;   // (b*T + t)*Hg + h
    if (row >= nrows) return;
    const int h = (int)(row % Hg);
    float wr[9][8], b0[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int c = 8 * cv + k;
        b0[k] = bias ? bias[c] : 0.f;
#pragma unroll
        for (int tp = 0; tp < 9; ++tp) wr[tp][k] = wgt[(size_t)c * 9 + tp];
    }
    const T *base = x + (row * Wg) * (long long)C + 8 * cv;  // token (b, t, h, 0)
    const long long rstride = (long long)Wg * C;            // one row of tokens
    float win[3][3][8];                                     // [row dh][column dw][channel]
    auto load_col = [&](int col, int slot) {
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            const int hh = h + a - 1;
            if (col >= 0 && col < Wg && hh >= 0 && hh < Hg) load8(base + (a - 1) * rstride + (long long)col * C, win[a][slot]);
            else zero8(win[a][slot]);
        }
    };
    load_col(-1, 0);
    load_col(0, 1);
    for (int w0 = 0; w0 < Wg; ++w0) {
        load_col(w0 + 1, 2);
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = b0[k];
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int l = 0; l < 3; ++l)
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[k] = fmaf(wr[a * 3 + l][k], win[a][l][k], acc[k]);
        store8(y + (row * Wg + w0) * (long long)C + 8 * cv, acc);
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                win[a][0][k] = win[a][1][k];
                win[a][1][k] = win[a][2][k];
            }
    }
}

// 3x1x1: one CTA per (b, h, w) position and block of kCThreads channel
// vectors; each thread slides a 3-frame window along t (one new load per output).
template <typename T>
__global__ void __launch_bounds__(kCThreads)
dwconv_temporal_kernel(const T *__restrict__ x, T *__restrict__ y, const float *__restrict__ wgt,
                       const float *__restrict__ bias, long long npos, int Tf, int Hg, int Wg, int C) {
    const int cv = blockIdx.x * kCThreads + threadIdx.x;
    if (8 * cv >= C) return;
    const long long pos = (long long)blockIdx.z * 65535 + blockIdx.y;   // b*Hg*Wg + h*Wg + w
    if (pos >= npos) return;
    const long long hw = (long long)Hg * Wg;
    const long long b = pos / hw, rem = pos % hw;
    float wr[3][8], b0[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int c = 8 * cv + k;
        b0[k] = bias ? bias[c] : 0.f;
#pragma unroll
        for (int tp = 0; tp < 3; ++tp) wr[tp][k] = wgt[(size_t)c * 3 + tp];
    }
    const long long fstride = hw * C;                       // one frame of tokens
    const T *base = x + (b * Tf * hw + rem) * C + 8 * cv;   // token (b, 0, h, w)
    T *obase = y + (b * Tf * hw + rem) * C + 8 * cv;
    // four outputs per step: frames t0 .. t0+3 from slots 0..5 (t0-1 .. t0+4),
    // the four new frames loaded together
    constexpr int kU = 4;
    float win[kU + 2][8];
    zero8(win[0]);
    load8(base, win[1]);
    for (int t0 = 0; t0 < Tf; t0 += kU) {
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (t0 + 1 + u < Tf) load8(base + (t0 + 1 + u) * fstride, win[2 + u]);
            else zero8(win[2 + u]);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (t0 + u >= Tf) break;
            float acc[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                acc[k] = fmaf(wr[2][k], win[u + 2][k], fmaf(wr[1][k], win[u + 1][k], fmaf(wr[0][k], win[u][k], b0[k])));
            store8(obase + (t0 + u) * fstride, acc);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            win[0][k] = win[kU][k];
            win[1][k] = win[kU + 1][k];
        }
    }
}

}  // namespace

int launch_dwconv(int is_bf16, const void *x, void *y, const float *w, const float *bias, int B, int T, int Hg,
                  int Wg, int C, int kt, int kh, int kw, cudaStream_t s) {
    // grid: x = channel blocks (fastest, so the blocks of one token row run
    // together), y and z = rows or positions (y < 65535)
    const long long gc = ((long long)C / 8 + kCThreads - 1) / kCThreads;
    if (gc > 0x7fffffffLL) return -1;
    auto grid_of = [&](long long n) { return dim3((unsigned)gc, (unsigned)(n < 65535 ? n : 65535), (unsigned)((n + 65534) / 65535)); };
    if (kt == 1 && kh == 3 && kw == 3) {
        const long long nrow = (long long)B * T * Hg;
        if (nrow <= 0 || nrow > 65535LL * 65535LL) return -1;
        const dim3 grid = grid_of(nrow);
        if (is_bf16)
            dwconv_spatial_kernel<__nv_bfloat16><<<grid, kCThreads, 0, s>>>(
                static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(y), w, bias, nrow, Hg, Wg, C);
        else
            dwconv_spatial_kernel<float><<<grid, kCThreads, 0, s>>>(static_cast<const float *>(x),
                                                                   static_cast<float *>(y), w, bias, nrow, Hg, Wg, C);
        return cudaGetLastError() == cudaSuccess ? 1 : -1;
    }
    if (kt == 3 && kh == 1 && kw == 1) {
        const long long npos = (long long)B * Hg * Wg;
        if (npos <= 0 || npos > 65535LL * 65535LL) return -1;
        const dim3 grid = grid_of(npos);
        if (is_bf16)
            dwconv_temporal_kernel<__nv_bfloat16><<<grid, kCThreads, 0, s>>>(
                static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(y), w, bias, npos, T, Hg, Wg, C);
        else
            dwconv_temporal_kernel<float><<<grid, kCThreads, 0, s>>>(static_cast<const float *>(x),
                                                                    static_cast<float *>(y), w, bias, npos, T, Hg, Wg, C);
        return cudaGetLastError() == cudaSuccess ? 1 : -1;
    }
    return -2;   // not a Mix-FFN kernel shape
}

}  // namespace la
