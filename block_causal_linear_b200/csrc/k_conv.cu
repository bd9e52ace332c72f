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
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "la_internal.cuh"
#include "la_sm100.cuh"

namespace la {
namespace {

using namespace sm100;

// Raised by a bounded wait of this file's kernels that gave up (0x100 | where);
// read by la_device_status through read_and_clear_conv_flag.
__device__ unsigned int g_wait_flag = 0;

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

// ---------------------------------------------------------------- bf16 on TMA tiles
//
// One CTA per tile of 64 channels (one 128-byte row of a TMA box): a single
// TMA load brings the tile's inputs with their halo into shared memory, the
// copy itself zero-filling the rows, columns and frames outside the tensor
// (the convolution's padding); the stencil is then read from shared memory
// with a sliding register window and each output vector of 8 channels is
// written with one 16-byte store (a warp writes 4 tokens x 128 contiguous
// bytes).  Input bytes come from DRAM once, plus the halo of neighbouring
// tiles (none when a tile is a whole frame or all frames).

constexpr int kTC = 64;             // channels per tile
constexpr int kTThreads = 256;
constexpr int kTSmemMax = 96 * 1024;   // tile budget: two CTAs per SM
constexpr int kTSeg = 8;            // outputs one thread slides through

// 8 bf16 channels from shared memory as 4 fp32 pairs (channels 2m, 2m + 1).
__device__ __forceinline__ void lds8x2(const uint8_t *p, float2 (&v)[4]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) v[m] = make_float2(__uint_as_float(w[m] << 16), __uint_as_float(w[m] & 0xFFFF0000u));
}

__device__ __forceinline__ void store8x2(__nv_bfloat16 *p, const float2 (&v)[4]) {
    *reinterpret_cast<uint4 *>(p) =
        make_uint4(bf2c(v[0].x, v[0].y), bf2c(v[1].x, v[1].y), bf2c(v[2].x, v[2].y), bf2c(v[3].x, v[3].y));
}

__device__ __forceinline__ void lds8(const uint8_t *p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

// 1x3x3: tile = output rows [h0, h0 + RH) x columns [w0, w0 + WT) of frame bt;
// shared memory holds rows h0-1 .. h0+RH and columns w0-1 .. w0+WT.
__global__ void __launch_bounds__(kTThreads, 2)
dwconv_spatial_tma_kernel(const __grid_constant__ CUtensorMap tm, __nv_bfloat16 *__restrict__ y,
                          const float *__restrict__ wgt, const float *__restrict__ bias, int Hg, int Wg, int C,
                          int RH, int WT, int ntw) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tile = align1024(smem_raw);
    __shared__ uint64_t bar;
    __shared__ int abort_word;
    const int tid = threadIdx.x;
    const int c0 = blockIdx.x * kTC;
    const int h0 = (blockIdx.y / ntw) * RH, w0 = (blockIdx.y % ntw) * WT;
    const int bt = blockIdx.z;
    const int rh = min(RH, Hg - h0), wt = min(WT, Wg - w0);
    const int tcols = WT + 2;
    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_word = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)((RH + 2) * tcols * kTC * 2));
        tma_load_4d(tile, &tm, &bar, c0, w0 - 1, h0 - 1, bt);
    }
    // the taps and bias of this thread's 8 channels while the tile comes in
    const int cv = tid & 7, c = c0 + 8 * cv;
    const bool live = c < C;
    float2 wr[9][4], b0[4];   // channel pairs (c + 2m, c + 2m + 1)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        b0[m] = live && bias ? make_float2(bias[c + 2 * m], bias[c + 2 * m + 1]) : make_float2(0.f, 0.f);
#pragma unroll
        for (int tp = 0; tp < 9; ++tp)
            wr[tp][m] = live ? make_float2(wgt[(size_t)(c + 2 * m) * 9 + tp], wgt[(size_t)(c + 2 * m + 1) * 9 + tp])
                             : make_float2(0.f, 0.f);
    }
    const bool ok = mbar_wait(&bar, 0, &abort_word, &g_wait_flag, 1);
    if (ok && live) {
        const int nseg = (wt + kTSeg - 1) / kTSeg;
        for (int item = tid >> 3; item < rh * nseg; item += kTThreads / 8) {
            const int r = item / nseg, wa = (item % nseg) * kTSeg;
            const int wb = min(wa + kTSeg, wt);
            // tile row r + a is input row h0 + r + a - 1; tile column j is input column w0 + j - 1.
            // Column j feeds outputs j - 2 (tap l = 2), j - 1 (l = 1) and j (l = 0): three
            // running sums, the oldest complete after each column (taps in column order).
            const uint8_t *src = tile + (size_t)r * tcols * (kTC * 2) + 16 * cv;
            __nv_bfloat16 *dst = y + (((size_t)bt * Hg + h0 + r) * Wg + w0 + wa) * C + c;
            // acc[jj % 3] starts output wa + jj; the three roles rotate (the loop is unrolled)
            float2 acc[3][4];
#pragma unroll
            for (int q = 0; q < 3; ++q)
#pragma unroll
                for (int m = 0; m < 4; ++m) acc[q][m] = make_float2(0.f, 0.f);
#pragma unroll
            for (int jj = 0; jj < kTSeg + 2; ++jj) {
                if (wa + jj < wb + 2) {
                    float2(&A)[4] = acc[(jj + 1) % 3];   // output wa + jj - 2: its last column
                    float2(&Bm)[4] = acc[(jj + 2) % 3];  // output wa + jj - 1
                    float2(&Cn)[4] = acc[jj % 3];        // output wa + jj: its first column
#pragma unroll
                    for (int m = 0; m < 4; ++m) Cn[m] = b0[m];
#pragma unroll
                    for (int a = 0; a < 3; ++a) {
                        float2 v[4];
                        lds8x2(src + ((size_t)a * tcols + wa + jj) * (kTC * 2), v);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            A[m] = ffma2(wr[a * 3 + 2][m], v[m], A[m]);
                            Bm[m] = ffma2(wr[a * 3 + 1][m], v[m], Bm[m]);
                            Cn[m] = ffma2(wr[a * 3 + 0][m], v[m], Cn[m]);
                        }
                    }
                    if (jj >= 2) {   // output wa + jj - 2 is complete
                        store8x2(dst, A);
                        dst += C;
                    }
                }
            }
        }
    }
    if (!ok && tid == 0) final_wait(&bar, 0);   // the copy may still be writing shared memory
}

// 3x1x1: tile = frames [t0, t0 + TT) x columns [w0, w0 + WT) of row h of batch b;
// shared memory holds frames t0-1 .. t0+TT of those columns.
__global__ void __launch_bounds__(kTThreads, 2)
dwconv_temporal_tma_kernel(const __grid_constant__ CUtensorMap tm, __nv_bfloat16 *__restrict__ y,
                           const float *__restrict__ wgt, const float *__restrict__ bias, int Tf, int Hg, int Wg,
                           int C, int TT, int WT, int ntw, int ntt) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tile = align1024(smem_raw);
    __shared__ uint64_t bar;
    __shared__ int abort_word;
    const int tid = threadIdx.x;
    const int c0 = blockIdx.x * kTC;
    int id = blockIdx.y;
    const int tw = id % ntw; id /= ntw;
    const int tt = id % ntt; id /= ntt;
    const int h = id;
    const int b = blockIdx.z;
    const int w0 = tw * WT, t0 = tt * TT;
    const int wt = min(WT, Wg - w0), nt = min(TT, Tf - t0);
    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_word = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)((TT + 2) * WT * kTC * 2));
        tma_load_5d(tile, &tm, &bar, c0, w0, h, t0 - 1, b);
    }
    const int cv = tid & 7, c = c0 + 8 * cv;
    const bool live = c < C;
    float2 wr[3][4], b0[4];   // channel pairs (c + 2m, c + 2m + 1)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        b0[m] = live && bias ? make_float2(bias[c + 2 * m], bias[c + 2 * m + 1]) : make_float2(0.f, 0.f);
#pragma unroll
        for (int tp = 0; tp < 3; ++tp)
            wr[tp][m] = live ? make_float2(wgt[(size_t)(c + 2 * m) * 3 + tp], wgt[(size_t)(c + 2 * m + 1) * 3 + tp])
                             : make_float2(0.f, 0.f);
    }
    const bool ok = mbar_wait(&bar, 0, &abort_word, &g_wait_flag, 2);
    if (ok && live) {
        const size_t fbytes = (size_t)WT * kTC * 2;   // one frame of the tile
        const size_t fstride = (size_t)Hg * Wg * C;   // one frame of y
        const int nseg = (nt + kTSeg - 1) / kTSeg;
        for (int item = tid >> 3; item < wt * nseg; item += kTThreads / 8) {
            const int w = item / nseg, ta = (item % nseg) * kTSeg;
            const int tb = min(ta + kTSeg, nt);
            // tile frame j is input frame t0 + j - 1
            const uint8_t *src = tile + (size_t)ta * fbytes + (size_t)w * (kTC * 2) + 16 * cv;
            // win[q % 3] holds tile frame ta + q; the roles rotate (the loop is unrolled)
            float2 win[3][4];
            lds8x2(src, win[0]);
            lds8x2(src + fbytes, win[1]);
            __nv_bfloat16 *dst = y + ((((size_t)b * Tf + t0 + ta) * Hg + h) * Wg + w0 + w) * C + c;
#pragma unroll
            for (int q = 0; q < kTSeg; ++q) {
                if (ta + q < tb) {
                    lds8x2(src + (size_t)(q + 2) * fbytes, win[(q + 2) % 3]);
                    float2 acc[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        acc[m] = ffma2(wr[2][m], win[(q + 2) % 3][m],
                                       ffma2(wr[1][m], win[(q + 1) % 3][m], ffma2(wr[0][m], win[q % 3][m], b0[m])));
                    store8x2(dst, acc);
                    dst += fstride;
                }
            }
        }
    }
    if (!ok && tid == 0) final_wait(&bar, 0);
}

// Balanced tiling of n into pieces of at most m: (pieces, size).
void tile_of(int n, int m, int &pieces, int &size) {
    if (m < 1) m = 1;
    pieces = (n + m - 1) / m;
    size = (n + pieces - 1) / pieces;
}

bool tma_smem_ready() {
    static std::once_flag once;
    static bool ok = false;
    std::call_once(once, [] {
        ok = set_smem((const void *)dwconv_spatial_tma_kernel, kTSmemMax + 1024) &&
             set_smem((const void *)dwconv_temporal_tma_kernel, kTSmemMax + 1024);
    });
    return ok;
}

// -1: could not launch; 0: shape not taken by the TMA kernels (the caller
// runs the plain ones); 1: launched.
int launch_dwconv_tma(const void *x, void *y, const float *w, const float *bias, int B, int T, int Hg, int Wg, int C,
                      bool spatial, cudaStream_t s) {
    if (C < kTC || !tc_available()) return 0;
    if (!tma_smem_ready()) return -1;
    const long long gc = (C + kTC - 1) / kTC;
    CUtensorMap m;
    const cuuint64_t es = 2;
    if (spatial) {
        int ntw, WT, nth, RH;
        tile_of(Wg, 254, ntw, WT);
        const int rowbytes = (WT + 2) * kTC * 2;
        const int rh_max = min(kTSmemMax / rowbytes - 2, 254);   // a box extent is at most 256
        if (rh_max < 1) return 0;
        tile_of(Hg, rh_max, nth, RH);
        const long long BT = (long long)B * T;
        if (BT > 65535 || (long long)nth * ntw > 65535 || gc > 0x7fffffffLL) return 0;
        const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)Wg, (cuuint64_t)Hg, (cuuint64_t)BT};
        const cuuint64_t strides[3] = {C * es, (cuuint64_t)Wg * C * es, (cuuint64_t)Hg * Wg * C * es};
        const cuuint32_t box[4] = {(cuuint32_t)kTC, (cuuint32_t)(WT + 2), (cuuint32_t)(RH + 2), 1};
        if (!make_bf16_map_nd(&m, x, 4, dims, strides, box)) return -1;
        const int smem = (RH + 2) * (WT + 2) * kTC * 2 + 1024;
        dwconv_spatial_tma_kernel<<<dim3((unsigned)gc, (unsigned)(nth * ntw), (unsigned)BT), kTThreads, smem, s>>>(
            m, static_cast<__nv_bfloat16 *>(y), w, bias, Hg, Wg, C, RH, WT, ntw);
        return cudaGetLastError() == cudaSuccess ? 1 : -1;
    }
    int ntw, WT, ntt, TT;
    tile_of(Wg, 32, ntw, WT);
    const int fbytes = WT * kTC * 2;
    const int tt_max = min(kTSmemMax / fbytes - 2, 254);
    if (tt_max < 1) return 0;
    tile_of(T, tt_max, ntt, TT);
    if (B > 65535 || (long long)Hg * ntt * ntw > 65535 || gc > 0x7fffffffLL) return 0;
    const cuuint64_t dims[5] = {(cuuint64_t)C, (cuuint64_t)Wg, (cuuint64_t)Hg, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[4] = {C * es, (cuuint64_t)Wg * C * es, (cuuint64_t)Hg * Wg * C * es,
                                   (cuuint64_t)T * Hg * Wg * C * es};
    const cuuint32_t box[5] = {(cuuint32_t)kTC, (cuuint32_t)WT, 1, (cuuint32_t)(TT + 2), 1};
    if (!make_bf16_map_nd(&m, x, 5, dims, strides, box)) return -1;
    const int smem = (TT + 2) * WT * kTC * 2 + 1024;
    dwconv_temporal_tma_kernel<<<dim3((unsigned)gc, (unsigned)(Hg * ntt * ntw), (unsigned)B), kTThreads, smem, s>>>(
        m, static_cast<__nv_bfloat16 *>(y), w, bias, T, Hg, Wg, C, TT, WT, ntw, ntt);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

int read_and_clear_conv_flag(unsigned *flag_out) {
    unsigned zero = 0;
    if (cudaMemcpyFromSymbol(flag_out, g_wait_flag, sizeof(unsigned)) != cudaSuccess) return -1;
    if (*flag_out && cudaMemcpyToSymbol(g_wait_flag, &zero, sizeof(unsigned)) != cudaSuccess) return -1;
    return 0;
}

int launch_dwconv(int is_bf16, const void *x, void *y, const float *w, const float *bias, int B, int T, int Hg,
                  int Wg, int C, int kt, int kh, int kw, cudaStream_t s) {
    // grid: x = channel blocks (fastest, so the blocks of one token row run
    // together), y and z = rows or positions (y < 65535)
    const long long gc = ((long long)C / 8 + kCThreads - 1) / kCThreads;
    if (gc > 0x7fffffffLL) return -1;
    auto grid_of = [&](long long n) { return dim3((unsigned)gc, (unsigned)(n < 65535 ? n : 65535), (unsigned)((n + 65534) / 65535)); };
    const bool sp = kt == 1 && kh == 3 && kw == 3, tp = kt == 3 && kh == 1 && kw == 1;
    if (is_bf16 && (sp || tp)) {
        const int r = launch_dwconv_tma(x, y, w, bias, B, T, Hg, Wg, C, sp, s);
        if (r != 0) return r;
    }
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
