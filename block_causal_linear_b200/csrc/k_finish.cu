// k_finish.cu -- state combine: fixed-order split sum, prefix over blocks,
// commit.
//
// Per (b, h), in a fixed order (so that results are reproducible bit for bit):
//   run = S_prior (or 0)                                   [S | Z], 1056 floats
//   for block n = 0 .. nb-1:
//       run += partial[n][0] + partial[n][1] + ... + partial[n][P-1]
//       S_eff[n] = run
// and, on commit, S <- S_eff[nb-1], Z likewise.  This is the cumulative state
// of the pages: KV_{1-2} = KV_1 + KV_2, and so on until the global KV
// ("Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı", section
// "Sabit Bellekli KV önbelleğe alma mekanizması", paragraph 4; sd114.wiki,
// "两大核心技术突破" item 2: one cumulative state, updated block by block).
//
// For the tensor-core apply it also packs S_eff into the bf16 MMA operand
// B (K = 32 key features x N = 48 columns: 32 value columns of S, Z, zeros) as
// a hi part and a lo part, hi = bf16(x), lo = bf16(x - hi), so that the MMA
// sees S_eff to about 16 mantissa bits.  Layout: K-major, no swizzle, core
// matrices of 8 rows x 16 bytes; element (n, k) at byte
//   (n / 8) * 512 + (k / 8) * 128 + (n % 8) * 16 + (k % 8) * 2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kFinThreads = 256;

__device__ __forceinline__ int op_offset(int nrow, int kcol) {
    return (nrow >> 3) * 512 + (kcol >> 3) * 128 + (nrow & 7) * 16 + (kcol & 7) * 2;
}

__global__ void __launch_bounds__(kFinThreads)
finish_kernel(const float *__restrict__ partials, float *__restrict__ seff,
              unsigned char *__restrict__ bop, float *__restrict__ S, float *__restrict__ Z,
              Plan p, int write_bop) {
    const int bh = blockIdx.x;
    for (int e = threadIdx.x; e < kKVZ; e += kFinThreads) {
        float run = 0.f;
        if (p.has_state) run = e < kD * kD ? S[(size_t)bh * kD * kD + e] : Z[(size_t)bh * kD + e - kD * kD];
        const int nrow = e < kD * kD ? (e % kD) : kD;     // value column, or the Z column
        const int kcol = e < kD * kD ? (e / kD) : (e - kD * kD);
        for (int n = 0; n < p.nb; ++n) {
            const float *src = partials + ((size_t)bh * p.nb + n) * p.P * kKVZ + e;
            for (int sp = 0; sp < p.P; ++sp) run += src[(size_t)sp * kKVZ];
            seff[((size_t)bh * p.nb + n) * kKVZ + e] = run;
            if (write_bop) {
                unsigned char *dst = bop + ((size_t)bh * p.nb + n) * 2 * kOpBytes + op_offset(nrow, kcol);
                const __nv_bfloat16 hi = __float2bfloat16_rn(run);
                const __nv_bfloat16 lo = __float2bfloat16_rn(run - __bfloat162float(hi));
                *reinterpret_cast<__nv_bfloat16 *>(dst) = hi;
                *reinterpret_cast<__nv_bfloat16 *>(dst + kOpBytes) = lo;
            }
        }
        if (p.commit) {
            if (e < kD * kD) S[(size_t)bh * kD * kD + e] = run;
            else Z[(size_t)bh * kD + e - kD * kD] = run;
        }
    }
    if (write_bop) {
        // rows 33..47 of the operand are zero (N padded to a multiple of 16)
        const int zrows = kOpRows - kD - 1;
        for (int w = threadIdx.x; w < p.nb * zrows * kD; w += kFinThreads) {
            const int n = w / (zrows * kD);
            const int nrow = kD + 1 + (w / kD) % zrows;
            const int kcol = w % kD;
            unsigned char *dst = bop + ((size_t)bh * p.nb + n) * 2 * kOpBytes + op_offset(nrow, kcol);
            *reinterpret_cast<unsigned short *>(dst) = 0;
            *reinterpret_cast<unsigned short *>(dst + kOpBytes) = 0;
        }
    }
}

}  // namespace

int launch_finish(const float *partials, float *seff, void *bop, float *S, float *Z, const Plan &p,
                  int write_bop, cudaStream_t s) {
    const long long grid = (long long)p.B * p.H;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    finish_kernel<<<(unsigned)grid, kFinThreads, 0, s>>>(partials, seff, static_cast<unsigned char *>(bop),
                                                       S, Z, p, write_bop);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace la
