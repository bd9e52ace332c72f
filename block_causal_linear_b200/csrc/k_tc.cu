// k_tc.cu -- tensor-core (tcgen05 + TMA) reduce and apply kernels for bf16.
//
// reduce: KV_n = sum_t phi(k_t)^T v_t and z_n = sum_t phi(k_t) over one split
//   of a block, for 4 heads at a time ("KV product then accumulate",
//   "Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı", section
//   "Sabit Bellekli KV önbelleğe alma mekanizması").  The contraction over
//   tokens is one M=128 x N=128 x K=16 MMA per 16 tokens: A = phi(K) of 4
//   heads (M = 4 x 32 key features, stored MN-major as TMA lands it), B = V of
//   the same 4 heads (N = 4 x 32 value features).  Only the 4 diagonal 32x32
//   blocks of D are used.  z comes from a second MMA against a 16-column
//   matrix of ones.  fp32 accumulation in TMEM across the whole split.
// apply: out_t = phi(q_t) S_eff / (phi(q_t) . Z_eff + eps) for 128-token tiles
//   of 2 heads: per head one M=128 x N=48 x K=32 contraction of phi(Q) against
//   the packed [S | Z | 0] operand, as a hi and a lo bf16 part accumulated in
//   the same TMEM columns (S_eff is carried to ~16 mantissa bits); the epilogue
//   divides, rounds to bf16 and stores with TMA.
//
// Both kernels: 6 warps; warp 0 issues TMA, warp 1 owns TMEM and issues the
// MMAs, warps 2..5 apply phi = ReLU in shared memory and run the epilogue.
// Every wait is bounded (la_sm100.cuh); a wait that gives up raises the device
// flag read by la_device_status and the CTA drains and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <utility>

#include "la_internal.cuh"
#include "la_sm100.cuh"

namespace la {

using namespace sm100;

// Raised by a bounded device-side wait that gave up (0x100 | where).
__device__ unsigned int g_wait_flag = 0;

namespace {

constexpr int kThreads = 192;   // 6 warps
constexpr int kWarpTma = 0;
constexpr int kWarpMma = 1;
constexpr int kWork = 128;      // threads of warps 2..5
constexpr uint32_t kTmemCols = 256;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ uint32_t relu2(uint32_t x) {
    // two bf16 in one word: as signed 16-bit integers every negative bf16
    // (sign bit set, including -0) is below 0, so a signed max with 0 is ReLU
    return __vmaxs2(x, 0u);
}

// Drain at exit after an abort: wait (briefly, ignoring the abort word) for
// anything still writing this CTA's shared memory or TMEM.
__device__ __forceinline__ void final_wait(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 0; i < (1u << 24); ++i) {
        if (mbar_try_wait(bar, parity)) return;
        if ((i & 255u) == 0 && global_timer_ns() - t0 > 200000000ull) return;
    }
}

// ================================================================ reduce

constexpr int kRStages = 3;
constexpr int kRBox = 64 * 128;             // [64 rows][64 bf16] = 8 KiB
constexpr int kRStageBytes = 4 * kRBox;     // k: 2 boxes (4 heads), v: 2 boxes
constexpr int kROnesOff = kRStages * kRStageBytes;
constexpr int kRBarOff = kROnesOff + 512;
constexpr int kRSmem = kRBarOff + (3 * kRStages + 1) * 8 + 16 + 1024;

__global__ void __launch_bounds__(kThreads, 2)
reduce_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 float *__restrict__ partials, const Plan p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *ones = smem + kROnesOff;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kRBarOff);
    uint64_t *relu_done = full + kRStages;
    uint64_t *empty = relu_done + kRStages;
    uint64_t *acc_ready = empty + kRStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_ready + 1);
    volatile int *abort_word = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int G = p.H / 4;
    long long id = blockIdx.x;
    const int g = (int)(id % G); id /= G;
    const int sp = (int)(id % p.P); id /= p.P;
    const int n = (int)(id % p.nb); id /= p.nb;
    const int b = (int)id;
    const long long blk0 = (long long)n * p.L;
    const long long blk1 = blk0 + p.L < p.N ? blk0 + p.L : (long long)p.N;
    const long long t0 = blk0 + (long long)sp * p.chunk;
    const long long t1 = t0 + p.chunk < blk1 ? t0 + p.chunk : blk1;
    const int nst = t1 > t0 ? (int)((t1 - t0 + 63) / 64) : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // k, v may come from the kernel just before this one: wait for it, then let
    // the next kernel (the state combine) be scheduled
    pdl_wait();
    pdl_trigger();

    if (nst == 0) {   // a split past the end of a short last block: its sums are zero
        for (int e = threadIdx.x; e < 4 * kKVZ; e += kThreads) {
            const int h = g * 4 + e / kKVZ;
            partials[((((size_t)b * p.H + h) * p.nb + n) * p.P + sp) * kKVZ + e % kKVZ] = 0.f;
        }
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&relu_done[s], kWork);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_ready, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    // B operand of the z contraction: 16 x 16 bf16 ones (any layout reads 1.0)
    for (int i = threadIdx.x; i < 128; i += kThreads) reinterpret_cast<uint32_t *>(ones)[i] = 0x3F803F80u;
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0;

    if (warp == kWarpTma) {
        if (lane == 0) {
            for (int i = 0; i < nst; ++i) {
                const int s = i % kRStages;
                const uint32_t ph = (uint32_t)(i / kRStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, &g_wait_flag, 1)) break;
                uint8_t *st = smem + s * kRStageBytes;
                mbar_arrive_expect_tx(&full[s], kRStageBytes);
                const int row = (int)(t0 + 64LL * i);
                const int c0 = g * 128;
                tma_load_3d(st + 0 * kRBox, &tm_k, &full[s], c0, row, b);
                tma_load_3d(st + 1 * kRBox, &tm_k, &full[s], c0 + 64, row, b);
                tma_load_3d(st + 2 * kRBox, &tm_v, &full[s], c0, row, b);
                tma_load_3d(st + 3 * kRBox, &tm_v, &full[s], c0 + 64, row, b);
                issued = i + 1;
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t id_kv = idesc_bf16(128, 128, 1, 1);
            const uint32_t id_z = idesc_bf16(128, 16, 1, 0);
            const uint64_t d_ones = smem_desc(smem_u32(ones), 128, 256, kLayoutNone);
            for (int i = 0; i < nst; ++i) {
                const int s = i % kRStages;
                const uint32_t ph = (uint32_t)(i / kRStages) & 1u;
                if (!mbar_wait(&relu_done[s], ph, abort_word, &g_wait_flag, 2)) break;
                tc_fence_after();
                const uint32_t kaddr = smem_u32(smem + s * kRStageBytes);
                const uint32_t vaddr = kaddr + 2 * kRBox;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    // MN-major, 128-byte swizzle: 64-wide MN atoms kRBox apart (LBO),
                    // 8-token groups 1024 B apart (SBO); 16 tokens = 2048 B per step
                    const uint64_t da = smem_desc(kaddr + kk * 2048, kRBox, 1024, kLayoutSw128);
                    const uint64_t db = smem_desc(vaddr + kk * 2048, kRBox, 1024, kLayoutSw128);
                    const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                    mma_bf16(tmem, da, db, id_kv, acc);
                    mma_bf16(tmem + 128, da, d_ones, id_z, acc);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(acc_ready);
        }
    } else {
        const int wt = threadIdx.x - 64;   // 0..127
        for (int i = 0; i < nst; ++i) {
            const int s = i % kRStages;
            const uint32_t ph = (uint32_t)(i / kRStages) & 1u;
            if (!mbar_wait(&full[s], ph, abort_word, &g_wait_flag, 3)) break;
            uint8_t *kt = smem + s * kRStageBytes;
            const long long row0 = t0 + 64LL * i;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = wt + 128 * j;           // 16-byte chunk of the two k boxes
                const int r = (c & 511) >> 3;         // token row inside its box
                uint4 *ptr = reinterpret_cast<uint4 *>(kt + (size_t)c * 16);
                uint4 x = *ptr;
                if (row0 + r < t1) {
                    x.x = relu2(x.x); x.y = relu2(x.y); x.z = relu2(x.z); x.w = relu2(x.w);
                } else {
                    x = make_uint4(0u, 0u, 0u, 0u);   // rows past the split contribute nothing
                }
                *ptr = x;
            }
            fence_proxy_async_smem();
            mbar_arrive(&relu_done[s]);
        }
        // epilogue: warp quarter q reads TMEM lanes 32q.. = key features of head 4g+q
        if (mbar_wait(acc_ready, 0, abort_word, &g_wait_flag, 4)) {
            __syncwarp();   // tcgen05.ld is warp-collective
            tc_fence_after();
            const int qd = warp & 3;
            const int h = g * 4 + qd;
            const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
            float kv[32];
            tmem_ld32(tmem + lane_off + 32 * qd, kv);
            const float z = tmem_ld1(tmem + lane_off + 128);
            tmem_wait_ld();
            float *dst = partials + ((((size_t)b * p.H + h) * p.nb + n) * p.P + sp) * kKVZ;
            float4 *drow = reinterpret_cast<float4 *>(dst + lane * kD);
#pragma unroll
            for (int j = 0; j < 8; ++j) drow[j] = make_float4(kv[4 * j], kv[4 * j + 1], kv[4 * j + 2], kv[4 * j + 3]);
            dst[kD * kD + lane] = z;
        }
    }

    // teardown: nothing may still write this CTA's shared memory or TMEM
    if (warp == kWarpTma && lane == 0 && *abort_word) {
        for (int i = issued - kRStages < 0 ? 0 : issued - kRStages; i < issued; ++i)
            final_wait(&full[i % kRStages], (uint32_t)(i / kRStages) & 1u);
    }
    if (warp == kWarpMma && lane == 0) final_wait(acc_ready, 0);
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ================================================================ apply

constexpr int kAStages = 3;
constexpr int kATile = 128 * 128;              // [128 rows][64 bf16] = 16 KiB: 2 heads
constexpr int kAOutOff = kAStages * kATile;    // 2 staging buffers for the TMA store
constexpr int kABopOff = kAOutOff + 2 * kATile;
constexpr int kABopBytes = 2 * 2 * kOpBytes;   // 2 heads x (hi, lo)
constexpr int kABarOff = kABopOff + kABopBytes;
constexpr int kASmem = kABarOff + (3 * kAStages + 6) * 8 + 16 + 1024;

__global__ void __launch_bounds__(kThreads, 2)
apply_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
                __nv_bfloat16 *__restrict__ out, const uint8_t *__restrict__ bop, const Plan p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stg = smem + kAOutOff;
    uint8_t *bops = smem + kABopOff;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kABarOff);
    uint64_t *relu_done = full + kAStages;
    uint64_t *empty = relu_done + kAStages;
    uint64_t *acc_full = empty + kAStages;      // [2]
    uint64_t *acc_empty = acc_full + 2;         // [2]
    uint64_t *bop_full = acc_empty + 2;
    uint64_t *drain = bop_full + 1;             // only used when a wait gave up
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_word = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int Gp = p.H / 2;
    long long id = blockIdx.x;
    const int hp = (int)(id % Gp); id /= Gp;
    const int spa = (int)(id % p.Pa); id /= p.Pa;
    const int n = (int)(id % p.nb); id /= p.nb;
    const int b = (int)id;
    const long long blk0 = (long long)n * p.L;
    const long long blk1 = blk0 + p.L < p.N ? blk0 + p.L : (long long)p.N;
    const long long ta0 = blk0 + (long long)spa * p.chunka;
    const long long ta1 = ta0 + p.chunka < blk1 ? ta0 + p.chunka : blk1;
    // the next kernel may be scheduled now: it waits for this grid before it
    // touches anything this grid reads or writes
    pdl_trigger();
    if (ta1 <= ta0) return;   // a split past the end of a short last block
    const int ntiles = (int)((ta1 - ta0 + 127) / 128);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&relu_done[s], kWork);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kWork);
        }
        mbar_init(bop_full, 1);
        mbar_init(drain, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_out);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0;
    bool bop_issued = false;

    if (warp == kWarpTma) {
        if (lane == 0) {
            // q is an input of the call, complete before the reduce of this call
            // started: its first tiles are fetched while the state combine still runs
            const int pre = ntiles < kAStages ? ntiles : kAStages;
            for (int i = 0; i < pre; ++i) {
                mbar_arrive_expect_tx(&full[i], kATile);
                tma_load_3d(smem + i * kATile, &tm_q, &full[i], hp * 64, (int)(ta0 + 128LL * i), b);
                issued = i + 1;
            }
            pdl_wait();   // the packed operand is written by the previous kernel
            mbar_arrive_expect_tx(bop_full, kABopBytes);
            for (int hh = 0; hh < 2; ++hh) {
                const size_t src = (((size_t)b * p.H + 2 * hp + hh) * p.nb + n) * 2 * kOpBytes;
                bulk_load(bops + hh * 2 * kOpBytes, bop + src, 2 * kOpBytes, bop_full);
            }
            bop_issued = true;
            for (int i = pre; i < ntiles; ++i) {
                const int s = i % kAStages;
                const uint32_t ph = (uint32_t)(i / kAStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, &g_wait_flag, 11)) break;
                mbar_arrive_expect_tx(&full[s], kATile);
                tma_load_3d(smem + s * kATile, &tm_q, &full[s], hp * 64, (int)(ta0 + 128LL * i), b);
                issued = i + 1;
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, kOpRows, 0, 0);
            const uint32_t baddr = smem_u32(bops);
            if (mbar_wait(bop_full, 0, abort_word, &g_wait_flag, 12)) {
                for (int i = 0; i < ntiles; ++i) {
                    const int s = i % kAStages;
                    const uint32_t ph = (uint32_t)(i / kAStages) & 1u;
                    const int ab = i & 1;
                    const uint32_t aph = (uint32_t)(i >> 1) & 1u;
                    if (!mbar_wait(&relu_done[s], ph, abort_word, &g_wait_flag, 13)) break;
                    if (!mbar_wait(&acc_empty[ab], aph ^ 1u, abort_word, &g_wait_flag, 14)) break;
                    tc_fence_after();
                    const uint32_t qaddr = smem_u32(smem + s * kATile);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t d = tmem + ab * 96 + hh * 48;
#pragma unroll
                        for (int part = 0; part < 2; ++part) {
#pragma unroll
                            for (int kk = 0; kk < 2; ++kk) {
                                // A: K-major, 128-byte swizzle; head hh is the 64-byte half
                                // of each 128-byte row, 16 features = 32 bytes per step
                                const uint64_t da = smem_desc(qaddr + hh * 64 + kk * 32, 16, 1024, kLayoutSw128);
                                // B: K-major, no swizzle, core matrices 128 B apart along K,
                                // 8-row groups 512 B apart; 16 features = 256 bytes per step
                                const uint64_t db = smem_desc(baddr + hh * 2 * kOpBytes + part * kOpBytes + kk * 256,
                                                              128, 512, kLayoutNone);
                                mma_bf16(d, da, db, idesc, (part | kk) ? 1u : 0u);
                            }
                        }
                    }
                    mma_commit(&empty[s]);
                    mma_commit(&acc_full[ab]);
                }
            }
        }
    } else {
        const int wt = threadIdx.x - 64;
        const int qd = warp & 3;
        const int r = 32 * qd + lane;               // token row of this thread in a tile
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        bool ok = true;

        auto relu_tile = [&](int i) -> bool {
            const int s = i % kAStages;
            const uint32_t ph = (uint32_t)(i / kAStages) & 1u;
            if (!mbar_wait(&full[s], ph, abort_word, &g_wait_flag, 15)) return false;
            uint8_t *qt = smem + s * kATile;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint4 *ptr = reinterpret_cast<uint4 *>(qt + (size_t)(wt + 128 * j) * 16);
                uint4 x = *ptr;
                x.x = relu2(x.x); x.y = relu2(x.y); x.z = relu2(x.z); x.w = relu2(x.w);
                *ptr = x;
            }
            fence_proxy_async_smem();
            mbar_arrive(&relu_done[s]);
            return true;
        };

        pdl_wait();   // every write to `out` comes after the previous kernel finished
        if (ntiles > 0) ok = relu_tile(0);
        for (int i = 0; i < ntiles && ok; ++i) {
            if (i + 1 < ntiles && !relu_tile(i + 1)) { ok = false; break; }
            const int ab = i & 1;
            const uint32_t aph = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(&acc_full[ab], aph, abort_word, &g_wait_flag, 16)) { ok = false; break; }
            __syncwarp();   // tcgen05.ld is warp-collective
            tc_fence_after();
            uint32_t packed[2][16];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float num[32];
                tmem_ld32(tmem + lane_off + ab * 96 + hh * 48, num);
                const float den = tmem_ld1(tmem + lane_off + ab * 96 + hh * 48 + kD);
                tmem_wait_ld();
                const float inv = 1.0f / (den + p.eps);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const __nv_bfloat162 t = __floats2bfloat162_rn(num[2 * j] * inv, num[2 * j + 1] * inv);
                    packed[hh][j] = *reinterpret_cast<const uint32_t *>(&t);
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);

            const long long row0 = ta0 + 128LL * i;
            const bool whole = row0 + 128 <= ta1 || ta1 == p.N;   // TMA clips rows >= N
            if (whole) {
                uint8_t *sb = stg + (i & 1) * kATile;
                if (wt == 0) bulk_wait_read<1>();   // the store of tile i-2 has read this buffer
                named_bar_sync(1, kWork);
#pragma unroll
                for (int c = 0; c < 8; ++c) {       // logical 16-byte chunk c: head c/4
                    const int pc = c ^ (r & 7);     // 128-byte swizzle
                    *reinterpret_cast<uint4 *>(sb + r * 128 + pc * 16) =
                        make_uint4(packed[c >> 2][4 * (c & 3)], packed[c >> 2][4 * (c & 3) + 1],
                                   packed[c >> 2][4 * (c & 3) + 2], packed[c >> 2][4 * (c & 3) + 3]);
                }
                fence_proxy_async_smem();
                named_bar_sync(1, kWork);
                if (wt == 0) {
                    tma_store_3d(&tm_out, sb, hp * 64, (int)row0, b);
                    bulk_commit();
                }
            } else if (row0 + r < ta1) {
                // a short last tile inside the tensor: the rows after ta1 belong to another block
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out + (((size_t)b * p.N + row0 + r) * p.H + 2 * hp + hh) * kD);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        dst[c] = make_uint4(packed[hh][4 * c], packed[hh][4 * c + 1], packed[hh][4 * c + 2],
                                            packed[hh][4 * c + 3]);
                }
            }
        }
        if (wt == 0) bulk_wait_all();
    }

    if (warp == kWarpTma && lane == 0 && *abort_word) {
        if (bop_issued) final_wait(bop_full, 0);
        for (int i = issued - kAStages < 0 ? 0 : issued - kAStages; i < issued; ++i)
            final_wait(&full[i % kAStages], (uint32_t)(i / kAStages) & 1u);
    }
    if (warp == kWarpMma && lane == 0 && *abort_word) {
        // make every MMA issued so far finish before TMEM is released
        mma_commit(drain);
        final_wait(drain, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ================================================================ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3D view of a [B][N][H*32] bf16 tensor, boxes of 64 features x box_rows tokens,
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap *m, const void *base, int B, int N, int H, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t row_bytes = (cuuint64_t)H * kD * 2;
    cuuint64_t dims[3] = {(cuuint64_t)H * kD, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[2] = {row_bytes, row_bytes * (cuuint64_t)N};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with programmatic stream serialization (the kernel may start while
// the previous kernel of the stream drains; it orders itself with pdl_wait).
template <typename... KArgs, typename... Args>
bool launch_pdl(void (*kernel)(KArgs...), unsigned grid, int smem, cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess;
}

bool set_smem(const void *kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

}  // namespace

bool tc_available() {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
    return major == 10 && minor == 0 && encode_fn() != nullptr;
}

int launch_reduce_tc(const void *k, const void *v, float *partials, const Plan &p, cudaStream_t s) {
    static std::once_flag once;
    static bool smem_ok = false;
    std::call_once(once, [] { smem_ok = set_smem((const void *)reduce_tc_kernel, kRSmem); });
    if (!smem_ok) return -1;
    CUtensorMap mk, mv;
    if (!make_map(&mk, k, p.B, p.N, p.H, 64) || !make_map(&mv, v, p.B, p.N, p.H, 64)) return -1;
    const long long grid = (long long)p.B * (p.H / 4) * p.nb * p.P;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    return launch_pdl(reduce_tc_kernel, (unsigned)grid, kRSmem, s, mk, mv, partials, p) ? 1 : -1;
}

int launch_apply_tc(const void *q, void *out, const void *bop, const Plan &p, cudaStream_t s) {
    static std::once_flag once;
    static bool smem_ok = false;
    std::call_once(once, [] { smem_ok = set_smem((const void *)apply_tc_kernel, kASmem); });
    if (!smem_ok) return -1;
    CUtensorMap mq, mo;
    if (!make_map(&mq, q, p.B, p.N, p.H, 128) || !make_map(&mo, out, p.B, p.N, p.H, 128)) return -1;
    const long long grid = (long long)p.B * p.nb * p.Pa * (p.H / 2);
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    return launch_pdl(apply_tc_kernel, (unsigned)grid, kASmem, s, mq, mo, static_cast<__nv_bfloat16 *>(out),
                      static_cast<const uint8_t *>(bop), p)
               ? 1
               : -1;
}

int read_and_clear_device_flag(cudaStream_t s, unsigned *flag_out) {
    unsigned zero = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(flag_out, g_wait_flag, sizeof(unsigned)) != cudaSuccess) return -1;
    if (*flag_out && cudaMemcpyToSymbol(g_wait_flag, &zero, sizeof(unsigned)) != cudaSuccess) return -1;
    return 0;
}

}  // namespace la
