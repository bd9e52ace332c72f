// k_finish.cu -- state combine: fixed-order split sum, prefix over blocks,
// commit.
//
// Per (b, h) and each of the 1056 numbers of [S | Z], in a fixed order (so
// that results are reproducible bit for bit):
//   run = S_prior (or 0)
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
//
// One thread per number: the P partial loads of a block are issued together
// and then added in split order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kFinThreads = 256;
constexpr int kBatch = 32;         // partial loads in flight per thread (one round for P <= 32)
constexpr int kZeroRows = kOpRows - kD - 1;
constexpr int kPerBH = kKVZ + kZeroRows * kD;   // numbers + zero-padding entries per (b, h)

// STRIDED: the split sums sit at runtime strides (the ranks' gathered sums);
// otherwise at the workspace's own: split sp of (bh, n) at ((bh nb + n) P + sp) kKVZ.
template <bool STRIDED>
__global__ void __launch_bounds__(kFinThreads)
finish_kernel(const float *__restrict__ partials, float *__restrict__ seff,
              unsigned char *__restrict__ bop, float *__restrict__ S, float *__restrict__ Z,
              Plan p, int write_bop, long long part_bh_rt, long long part_sp_rt) {
    // the split sums of (bh, block n) start at part_bh * (bh nb + n): P slots of
    // the split plan, or skP slots of the RoPE kernels' stream-K plan
    const long long part_bh = STRIDED ? part_bh_rt : (long long)(p.sk_layout ? p.skP : p.P) * kKVZ;
    const long long part_sp = STRIDED ? part_sp_rt : (long long)kKVZ;
    // let the apply be scheduled now (it prefetches its q tiles), then wait
    // for the reduce before reading its partials
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const long long w = (long long)blockIdx.x * kFinThreads + threadIdx.x;
    const long long bh = w / kPerBH;
    const int e = (int)(w % kPerBH);
    if (bh >= (long long)p.B * p.H) return;

    if (e >= kKVZ) {   // zero rows 33..47 of the packed operand (N padded to 48)
        if (!write_bop) return;
        const int z = e - kKVZ;
        const int nrow = kD + 1 + z / kD, kcol = z % kD;
        for (int n = 0; n < p.nb; ++n) {
            unsigned char *dst = bop + ((size_t)bh * p.nb + n) * 2 * kOpBytes + op_offset(nrow, kcol);
            *reinterpret_cast<unsigned short *>(dst) = 0;
            *reinterpret_cast<unsigned short *>(dst + kOpBytes) = 0;
        }
        return;
    }

    float run = 0.f;
    if (p.has_state) run = e < kD * kD ? S[(size_t)bh * kD * kD + e] : Z[(size_t)bh * kD + e - kD * kD];
    const int nrow = e < kD * kD ? (e % kD) : kD;     // value column, or the Z column
    const int kcol = e < kD * kD ? (e / kD) : (e - kD * kD);
    for (int n = 0; n < p.nb; ++n) {
        // split sp of (bh, n) at partials + (bh * nb + n) * part_bh + sp * part_sp
        const float *src = partials + ((size_t)bh * p.nb + n) * part_bh + e;
        int P = p.P;
        if (!STRIDED && p.sk_layout) {
            // the CTAs of the stream-K plan that met unit (b, head group, n), in order
            const int b = (int)(bh / p.H), g = (int)(bh % p.H) / 4;
            const long long first = sk_unit_first(p.skr, b, n, g);
            P = sk_cta_of(p.skr, first + sk_len(p.skr, n) - 1) - sk_cta_of(p.skr, first) + 1;
        }
        for (int s0 = 0; s0 < P; s0 += kBatch) {
            float v[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) v[j] = s0 + j < P ? __ldg(src + (size_t)(s0 + j) * part_sp) : 0.f;
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                if (s0 + j < P) run += v[j];
        }
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

}  // namespace

namespace {
int launch_finish_strided(const float *partials, float *seff, void *bop, float *S, float *Z, const Plan &p,
                          int write_bop, long long part_bh, long long part_sp, cudaStream_t s) {
    const long long threads = (long long)p.B * p.H * kPerBH;
    const long long grid = (threads + kFinThreads - 1) / kFinThreads;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    // programmatic stream serialization: the kernel may start while the reduce
    // drains; it waits for it (griddepcontrol.wait) before reading anything
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kFinThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const bool strided = part_bh != (long long)(p.sk_layout ? p.skP : p.P) * kKVZ || part_sp != kKVZ;
    return cudaLaunchKernelEx(&cfg, strided ? finish_kernel<true> : finish_kernel<false>, partials, seff,
                              static_cast<unsigned char *>(bop), S, Z, p, write_bop, part_bh, part_sp) == cudaSuccess
               ? 1
               : -1;
}
}  // namespace

int launch_finish(const float *partials, float *seff, void *bop, float *S, float *Z, const Plan &p,
                  int write_bop, cudaStream_t s) {
    return launch_finish_strided(partials, seff, bop, S, Z, p, write_bop,
                                 (long long)(p.sk_layout ? p.skP : p.P) * kKVZ, kKVZ, s);
}



int launch_finish_ranks(const float *gathered, int R, float *seff, void *bop, float *S, float *Z, const Plan &p,
                        int write_bop, cudaStream_t s) {
    if (p.nb != 1 || R < 1) return -1;
    Plan q = p;
    q.P = R;   // the ranks' partial sums play the splits, in rank order
    q.sk_layout = 0;
    return launch_finish_strided(gathered, seff, bop, S, Z, q, write_bop, kKVZ, (long long)p.B * p.H * kKVZ,
                                 s);
}

}  // namespace la
