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
#include "la_rope.cuh"

namespace la {
namespace {

constexpr int kBThreads = 256;   // bwd_finish_kernel

// One token row (32 features of one head) between global memory and registers,
// in 16-byte pieces.
__device__ __forceinline__ void load_row(const float *p, float (&x)[kD]) {
#pragma unroll
    for (int i = 0; i < kD / 4; ++i) {
        const float4 v = reinterpret_cast<const float4 *>(p)[i];
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
}
__device__ __forceinline__ void load_row(const __nv_bfloat16 *p, float (&x)[kD]) {
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
        const uint4 v = reinterpret_cast<const uint4 *>(p)[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            x[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}
// Half a token row (16 features) between global memory and registers.
__device__ __forceinline__ void load_half(const float *p, float (&x)[kD / 2]) {
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
        const float4 v = reinterpret_cast<const float4 *>(p)[i];
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
}
__device__ __forceinline__ void load_half(const __nv_bfloat16 *p, float (&x)[kD / 2]) {
#pragma unroll
    for (int i = 0; i < kD / 16; ++i) {
        const uint4 v = reinterpret_cast<const uint4 *>(p)[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            x[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}
__device__ __forceinline__ void store_row(float *p, const float (&x)[kD]) {
#pragma unroll
    for (int i = 0; i < kD / 4; ++i)
        reinterpret_cast<float4 *>(p)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}
__device__ __forceinline__ uint32_t bf2(float a, float b) {
    const __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&t);
}
__device__ __forceinline__ void store_row(__nv_bfloat16 *p, const float (&x)[kD]) {
#pragma unroll
    for (int i = 0; i < kD / 8; ++i)
        reinterpret_cast<uint4 *>(p)[i] = make_uint4(bf2(x[8 * i], x[8 * i + 1]), bf2(x[8 * i + 2], x[8 * i + 3]),
                                                     bf2(x[8 * i + 4], x[8 * i + 5]), bf2(x[8 * i + 6], x[8 * i + 7]));
}
__device__ __forceinline__ void store_half(float *p, const float (&x)[kD / 2]) {
#pragma unroll
    for (int i = 0; i < kD / 8; ++i)
        reinterpret_cast<float4 *>(p)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}
__device__ __forceinline__ void store_half(__nv_bfloat16 *p, const float (&x)[kD / 2]) {
#pragma unroll
    for (int i = 0; i < kD / 16; ++i)
        reinterpret_cast<uint4 *>(p)[i] = make_uint4(bf2(x[8 * i], x[8 * i + 1]), bf2(x[8 * i + 2], x[8 * i + 3]),
                                                     bf2(x[8 * i + 4], x[8 * i + 5]), bf2(x[8 * i + 6], x[8 * i + 7]));
}

// cos, sin of the 16 feature pairs of token t of the call (numerator RoPE):
// the token's frame t_offset + t / (Hg Wg), row and column once (32-bit
// division by multiply-shift), then each pair's angle pos * theta along the
// pair's axis.
__device__ __forceinline__ void token_cs(const Plan &p, long long t, float (&c)[kD / 2], float (&s)[kD / 2]) {
    const Pos q = token_pos(p, (int)t);
    const int f = p.t_offset + q.f;
#pragma unroll
    for (int pr = 0; pr < kD / 2; ++pr) {
        const int ax = p.axis[pr];
        const int pos = ax == 0 ? f : (ax == 1 ? q.h : q.w);
        sincosf((float)pos * p.theta[pr], &s[pr], &c[pr]);
    }
}
// The same values read from the call's cos/sin table (built with the same
// sincosf of the same products): 8 records, one per group of 4 features.
__device__ __forceinline__ void token_cs_tab(const Plan &p, const uint8_t *tab, long long t, float (&c)[kD / 2],
                                             float (&s)[kD / 2]) {
    const Pos q = token_pos(p, (int)t);
#pragma unroll
    for (int m = 0; m < kD / 4; ++m) {
        const float4 r = tab_rec(tab, group_rec(p, m), q);
        c[2 * m] = r.x;
        c[2 * m + 1] = r.y;
        s[2 * m] = r.z;
        s[2 * m + 1] = r.w;
    }
}
// x <- R x (sgn = +1) or R^T x (sgn = -1), pair by pair.
__device__ __forceinline__ void rotate_row(float (&x)[kD], const float (&c)[kD / 2], const float (&s)[kD / 2],
                                           float sgn) {
#pragma unroll
    for (int pr = 0; pr < kD / 2; ++pr) {
        const float a = x[2 * pr], b = x[2 * pr + 1], sn = sgn * s[pr];
        x[2 * pr] = a * c[pr] - b * sn;
        x[2 * pr + 1] = a * sn + b * c[pr];
    }
}

constexpr int kQThreads = 128;
constexpr int kQRows = 64;               // token rows per round: two threads each
constexpr int kQStride = kD + 4;         // 36 floats: rows 16-byte aligned, 4 banks apart
constexpr int kQTab = 8192;              // the call's cos/sin table, when it fits
constexpr int kQSmem = (kKVZ + 3 * kQRows * kQStride + kQRows) * 4 + kQTab;

// One CTA per (b, h, block n, split sp): dq of the split's tokens and the
// split's [dS | dZ] sums.  seff: [B][H][nb][1056] inclusive prefix state.
// Per round of 64 tokens: two threads take each token (num, den, g, c, dq,
// half of the features each); then [dS | dZ] += [psi(q) g^T | c phi(q)] over
// the round's rows, each thread a 4 x 4 block of dS for half of the rows (the
// two halves are added in a fixed order at the end).
template <typename T>
__global__ void __launch_bounds__(kQThreads, 4)   // at most 128 registers: 4 CTAs per SM (measured best)
bwd_q_kernel(const T *__restrict__ q, const T *__restrict__ dout, const float *__restrict__ seff,
             T *__restrict__ dq, float *__restrict__ bpart, Plan p) {
    extern __shared__ __align__(16) float qsm[];
    float *Ss = qsm;                                  // S_n rows (key feature), then Z_n
    float *pq = Ss + kKVZ;                            // psi(q)  [kQRows][kQStride]
    float *fq = pq + kQRows * kQStride;               // phi(q)
    float *gg = fq + kQRows * kQStride;               // g = dout / den
    float *cc = gg + kQRows * kQStride;               // c = -(dout . num) / den^2

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
    for (int e = tid; e < kKVZ; e += kQThreads) Ss[e] = src[e];
    uint8_t *tab = reinterpret_cast<uint8_t *>(cc + kQRows);
    const bool use_tab = p.rope && p.tab_bytes > 0 && p.tab_bytes <= kQTab;
    if (use_tab) build_table(tab, p, tid, kQThreads);

    const int gi = tid >> 6, j = tid & 63;            // accumulation: row half, 4 x 4 block
    const int a0 = 4 * (j >> 3), c0 = 4 * (j & 7);
    float acc[4][4], accz[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        accz[i] = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) acc[i][k2] = 0.f;
    }
    __syncthreads();

    // Two threads per token (lanes 2i, 2i + 1 of a warp): each produces half
    // of num, g and dq (value columns, and key features, 16 hf ..), and the
    // halves of the two dot products are added in a fixed order (half 0, then
    // half 1) by both threads.
    const int tr = tid >> 1, hf = tid & 1;
    for (long long r0 = t0; r0 < t1; r0 += kQRows) {
        const long long t = r0 + tr;
        const bool valid = t < t1;
        const size_t off = (((size_t)b * p.N + (valid ? t : t0)) * p.H + h) * kD;
        float x[kD];
        uint32_t pos = 0;                              // bit a: q_a > 0
        if (valid) load_row(q + off, x);
#pragma unroll
        for (int a = 0; a < kD; ++a) {
            const float v = valid ? x[a] : 0.f;
            pos |= (v > 0.f ? 1u : 0u) << a;
            x[a] = fmaxf(v, 0.f);                      // phi(q)
        }
        // register arrays are indexed by constants only (a runtime half index
        // would put them in local memory): this thread's half by a select
        auto xh = [&](int a) { return hf ? x[16 + a] : x[a]; };
        float dh = 0.f;                                // phi(q) . Z over this thread's half
#pragma unroll
        for (int a = 0; a < kD / 2; ++a) dh = fmaf(xh(a), Ss[kD * kD + 16 * hf + a], dh);
        const float dx = __shfl_xor_sync(0xffffffffu, dh, 1);
        const float den = (hf ? dx + dh : dh + dx) + p.eps;
#pragma unroll
        for (int a = 0; a < kD / 2; a += 4)
            *reinterpret_cast<float4 *>(fq + tr * kQStride + 16 * hf + a) = make_float4(xh(a), xh(a + 1), xh(a + 2), xh(a + 3));
        float cs_c[kD / 2], cs_s[kD / 2];
        if (p.rope && valid) {
            if (use_tab) token_cs_tab(p, tab, t, cs_c, cs_s);
            else token_cs(p, t, cs_c, cs_s);
            rotate_row(x, cs_c, cs_s, 1.f);            // x is psi(q) from here on
        }
#pragma unroll
        for (int a = 0; a < kD / 2; a += 4)
            *reinterpret_cast<float4 *>(pq + tr * kQStride + 16 * hf + a) = make_float4(xh(a), xh(a + 1), xh(a + 2), xh(a + 3));
        // num = psi(q) S_n over this thread's 16 value columns
        float num[kD / 2];
#pragma unroll
        for (int c = 0; c < kD / 2; ++c) num[c] = 0.f;
#pragma unroll
        for (int a = 0; a < kD; ++a) {
            const float4 *row = reinterpret_cast<const float4 *>(Ss + a * kD + 16 * hf);
#pragma unroll
            for (int c4 = 0; c4 < kD / 8; ++c4) {
                const float4 sv = row[c4];
                num[4 * c4] = fmaf(x[a], sv.x, num[4 * c4]);
                num[4 * c4 + 1] = fmaf(x[a], sv.y, num[4 * c4 + 1]);
                num[4 * c4 + 2] = fmaf(x[a], sv.z, num[4 * c4 + 2]);
                num[4 * c4 + 3] = fmaf(x[a], sv.w, num[4 * c4 + 3]);
            }
        }
        float o[kD / 2];
        if (valid) load_half(dout + off + 16 * hf, o);
        float nh = 0.f;
#pragma unroll
        for (int c = 0; c < kD / 2; ++c) {
            if (!valid) o[c] = 0.f;
            nh = fmaf(o[c], num[c], nh);
        }
        const float nx = __shfl_xor_sync(0xffffffffu, nh, 1);
        const float dn = hf ? nx + nh : nh + nx;
        const float inv = 1.0f / den;
        const float cr = valid ? -dn * inv * inv : 0.f;
#pragma unroll
        for (int c = 0; c < kD / 2; ++c) o[c] *= inv;  // g, this thread's half
#pragma unroll
        for (int c = 0; c < kD / 2; c += 4)
            *reinterpret_cast<float4 *>(gg + tr * kQStride + 16 * hf + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        if (hf == 0) cc[tr] = cr;
        __syncwarp();                                  // the partner's half of g is in gg
        if (valid) {
            // dq = mask (R^T (S g) + c Z) over this thread's 16 key features
            float gv[kD];
#pragma unroll
            for (int c = 0; c < kD; c += 4) {
                const float4 gq = *reinterpret_cast<const float4 *>(gg + tr * kQStride + c);
                gv[c] = gq.x; gv[c + 1] = gq.y; gv[c + 2] = gq.z; gv[c + 3] = gq.w;
            }
            float dp[kD / 2];
#pragma unroll
            for (int a = 0; a < kD / 2; ++a) {
                const float4 *row = reinterpret_cast<const float4 *>(Ss + (16 * hf + a) * kD);
                float sacc = 0.f;
#pragma unroll
                for (int c4 = 0; c4 < kD / 4; ++c4) {
                    const float4 sv = row[c4];
                    sacc = fmaf(sv.x, gv[4 * c4], sacc);
                    sacc = fmaf(sv.y, gv[4 * c4 + 1], sacc);
                    sacc = fmaf(sv.z, gv[4 * c4 + 2], sacc);
                    sacc = fmaf(sv.w, gv[4 * c4 + 3], sacc);
                }
                dp[a] = sacc;
            }
            if (p.rope) {
#pragma unroll
                for (int pr = 0; pr < kD / 4; ++pr) {   // this half's pairs 8 hf + pr, by R^T
                    const float c = hf ? cs_c[8 + pr] : cs_c[pr], sn = hf ? cs_s[8 + pr] : cs_s[pr];
                    const float u = dp[2 * pr], w = dp[2 * pr + 1];
                    dp[2 * pr] = u * c + w * sn;
                    dp[2 * pr + 1] = -u * sn + w * c;
                }
            }
#pragma unroll
            for (int a = 0; a < kD / 2; ++a)
                dp[a] = (pos >> (16 * hf + a)) & 1u ? fmaf(cr, Ss[kD * kD + 16 * hf + a], dp[a]) : 0.f;
            store_half(dq + off + 16 * hf, dp);
        }
        __syncthreads();
        // [dS | dZ] over this thread's half of the round's rows, row order
        const int nr = t1 - r0 < kQRows ? (int)(t1 - r0) : kQRows;
        const int rb = gi * (kQRows / 2), re = rb + kQRows / 2 < nr ? rb + kQRows / 2 : nr;
        for (int r = rb; r < re; ++r) {
            const float4 pa = *reinterpret_cast<const float4 *>(pq + r * kQStride + a0);
            const float4 gc = *reinterpret_cast<const float4 *>(gg + r * kQStride + c0);
            const float pav[4] = {pa.x, pa.y, pa.z, pa.w}, gcv[4] = {gc.x, gc.y, gc.z, gc.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k2 = 0; k2 < 4; ++k2) acc[i][k2] = fmaf(pav[i], gcv[k2], acc[i][k2]);
            if (j < 8) {
                const float4 fz = *reinterpret_cast<const float4 *>(fq + r * kQStride + 4 * j);
                const float cr2 = cc[r];
                accz[0] = fmaf(cr2, fz.x, accz[0]);
                accz[1] = fmaf(cr2, fz.y, accz[1]);
                accz[2] = fmaf(cr2, fz.z, accz[2]);
                accz[3] = fmaf(cr2, fz.w, accz[3]);
            }
        }
        __syncthreads();
    }
    // the two row halves: first + second, in that order
    float *comb = pq;
    if (gi == 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) comb[(a0 + i) * kD + c0 + k2] = acc[i][k2];
        if (j < 8)
#pragma unroll
            for (int i = 0; i < 4; ++i) comb[kD * kD + 4 * j + i] = accz[i];
    }
    __syncthreads();
    if (gi == 0) {
        float *dst = bpart + ((bh * p.nb + n) * p.P + sp) * kKVZ;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
                const int e = (a0 + i) * kD + c0 + k2;
                dst[e] = acc[i][k2] + comb[e];
            }
        if (j < 8)
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[kD * kD + 4 * j + i] = accz[i] + comb[kD * kD + 4 * j + i];
    }
}

// One thread per (b, h, number e of [dS | dZ]): suffix sums over blocks, last
// block first, the P splits of a block in split order.
__global__ void __launch_bounds__(kBThreads)
bwd_finish_kernel(const float *__restrict__ bpart, float *__restrict__ G, unsigned char *__restrict__ gop, Plan p) {
    // the key-side kernel may be scheduled now (it prefetches its k, v tiles);
    // it waits for this grid before reading G
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const long long w = (long long)blockIdx.x * kBThreads + threadIdx.x;
    if (w >= (long long)p.B * p.H * kKVZ) return;
    const size_t bh = (size_t)(w / kKVZ);
    const int e = (int)(w % kKVZ);
    float run = 0.f;
    for (int n = p.nb - 1; n >= 0; --n) {
        const float *src = bpart + (bh * p.nb + n) * p.P * kKVZ + e;
        for (int s = 0; s < p.P; ++s) run += src[(size_t)s * kKVZ];
        G[(bh * p.nb + n) * kKVZ + e] = run;
        if (gop && e < kD * kD) {
            // bf16 hi + lo of G[a][c] as the B operands of the key side:
            // G (row c, K a) and G^T (row a, K c)
            const int a = e / kD, c = e % kD;
            unsigned char *o = gop + (bh * p.nb + n) * 4 * (size_t)kGopBytes;
            const __nv_bfloat16 hi = __float2bfloat16_rn(run);
            const __nv_bfloat16 lo = __float2bfloat16_rn(run - __bfloat162float(hi));
            *reinterpret_cast<__nv_bfloat16 *>(o + op_offset(c, a)) = hi;
            *reinterpret_cast<__nv_bfloat16 *>(o + kGopBytes + op_offset(c, a)) = lo;
            *reinterpret_cast<__nv_bfloat16 *>(o + 2 * kGopBytes + op_offset(a, c)) = hi;
            *reinterpret_cast<__nv_bfloat16 *>(o + 3 * kGopBytes + op_offset(a, c)) = lo;
        }
    }
}

constexpr int kKThreads = 128;

// One CTA per (b, block m, head h, tile of 128 tokens); one thread per token.
// Each row a of G_m (8 broadcast 16-byte loads) serves both products:
// dv += psi(k)_a G[a][:] and d psi(k)_a = G[a][:] . v.
template <typename T>
__global__ void __launch_bounds__(kKThreads)
bwd_k_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ G,
             T *__restrict__ dk, T *__restrict__ dv, Plan p) {
    __shared__ __align__(16) float Gs[kKVZ];
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
    const size_t off = (((size_t)b * p.N + t) * p.H + h) * kD;
    float ps[kD], vv[kD];
    load_row(k + off, ps);
    load_row(v + off, vv);
    uint32_t pos = 0;
#pragma unroll
    for (int a = 0; a < kD; ++a) {
        pos |= (ps[a] > 0.f ? 1u : 0u) << a;
        ps[a] = fmaxf(ps[a], 0.f);
    }
    float cs_c[kD / 2], cs_s[kD / 2];
    if (p.rope) {
        token_cs(p, t, cs_c, cs_s);
        rotate_row(ps, cs_c, cs_s, 1.f);
    }
    float dvv[kD], dp[kD];
#pragma unroll
    for (int c = 0; c < kD; ++c) dvv[c] = 0.f;
#pragma unroll 4
    for (int a = 0; a < kD; ++a) {
        const float4 *row = reinterpret_cast<const float4 *>(Gs + a * kD);
        float s = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < kD / 4; ++c4) {
            const float4 gv = row[c4];
            dvv[4 * c4] = fmaf(ps[a], gv.x, dvv[4 * c4]);
            dvv[4 * c4 + 1] = fmaf(ps[a], gv.y, dvv[4 * c4 + 1]);
            dvv[4 * c4 + 2] = fmaf(ps[a], gv.z, dvv[4 * c4 + 2]);
            dvv[4 * c4 + 3] = fmaf(ps[a], gv.w, dvv[4 * c4 + 3]);
            s = fmaf(gv.x, vv[4 * c4], s);
            s = fmaf(gv.y, vv[4 * c4 + 1], s);
            s = fmaf(gv.z, vv[4 * c4 + 2], s);
            s = fmaf(gv.w, vv[4 * c4 + 3], s);
        }
        dp[a] = s;
    }
    if (p.rope) rotate_row(dp, cs_c, cs_s, -1.f);
#pragma unroll
    for (int a = 0; a < kD; ++a) dp[a] = (pos >> a) & 1u ? dp[a] + Gs[kD * kD + a] : 0.f;
    store_row(dk + off, dp);
    store_row(dv + off, dvv);
}

}  // namespace

int launch_bwd_q(int is_bf16, const void *q, const void *dout, const float *seff, void *dq, float *bpart,
                 const Plan &p, cudaStream_t s) {
    const long long grid = (long long)p.B * p.H * p.nb * p.P;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    static const bool attrs = cudaFuncSetAttribute((const void *)bwd_q_kernel<__nv_bfloat16>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem) == cudaSuccess &&
                              cudaFuncSetAttribute((const void *)bwd_q_kernel<float>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem) == cudaSuccess;
    if (!attrs) return -1;
    if (is_bf16)
        bwd_q_kernel<__nv_bfloat16><<<(unsigned)grid, kQThreads, kQSmem, s>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(dout), seff,
            static_cast<__nv_bfloat16 *>(dq), bpart, p);
    else
        bwd_q_kernel<float><<<(unsigned)grid, kQThreads, kQSmem, s>>>(static_cast<const float *>(q),
                                                                 static_cast<const float *>(dout), seff,
                                                                 static_cast<float *>(dq), bpart, p);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_bwd_finish(const float *bpart, float *G, void *gop, const Plan &p, cudaStream_t s) {
    const long long threads = (long long)p.B * p.H * kKVZ;
    const long long grid = (threads + kBThreads - 1) / kBThreads;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    bwd_finish_kernel<<<(unsigned)grid, kBThreads, 0, s>>>(bpart, G, static_cast<unsigned char *>(gop), p);
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
