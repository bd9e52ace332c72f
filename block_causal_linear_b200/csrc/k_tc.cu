// k_tc.cu -- tensor-core (tcgen05 + TMA) reduce and apply kernels for bf16.
//
// reduce: KV_n = sum_t psi(k_t)^T v_t and z_n = sum_t phi(k_t) over one split
//   of a block, for 4 heads at a time ("KV product then accumulate",
//   "Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı", section
//   "Sabit Bellekli KV önbelleğe alma mekanizması").  The contraction over
//   tokens is one M=128 x N=128 x K=16 MMA per 16 tokens: A = psi(K) of 4
//   heads (M = 4 x 32 key features, stored MN-major as TMA lands it), B = V of
//   the same 4 heads (N = 4 x 32 value features).  Only the 4 diagonal 32x32
//   blocks of D are used.  fp32 accumulation in TMEM across the whole split.
//   z comes from a second MMA against a 16-column matrix of ones.
// apply: out_t = phi(q_t) S_eff / (phi(q_t) . Z_eff + eps) for 128-token tiles
//   of 2 heads: per head one M=128 x N=48 x K=32 contraction of phi(Q) against
//   the packed [S | Z | 0] operand, as a hi and a lo bf16 part accumulated in
//   the same TMEM columns.  The epilogue divides, rounds to bf16 and stores
//   with TMA.
// Calls with RoPE run the kernels of k_rope_tc.cu instead.
//
// Warp roles: warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs.  In the
// reduce, warps 2..5 apply phi = ReLU in shared memory and run the epilogue; in
// the apply, warps 6..9 transform the q tiles while warps 2..5 run the epilogue
// of the previous tile.  Every wait is bounded (la_sm100.cuh); a
// wait that gives up raises the device flag read by la_device_status and the
// CTA drains and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
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

constexpr int kWarpTma = 0;
constexpr int kWarpMma = 1;
constexpr int kWork = 128;      // threads of warps 2..5

// ---------------------------------------------------------------- NVFP4
// ReLU on 8 packed E2M1 codes: a code with its sign bit (bit 3 of the nibble)
// set is negative or -0, and becomes +0.
__device__ __forceinline__ uint32_t relu_e2m1x8(uint32_t w) {
    const uint32_t neg = (w >> 3) & 0x11111111u;
    return w & ~(neg * 15u);
}

// 16 E2M1 codes (8 bytes, element 2i in the low nibble) times their E4M3 block
// scale, as 16 f16 (features 0-7 in `a`, 8-15 in `b`).  Exact: a code value
// has 2 significant bits and a scale 4, so every product (0 or 2^-10 .. 2688)
// is an f16.
__device__ __forceinline__ void decode_nvfp4_16(uint2 c, uint8_t sf, uint4 &a, uint4 &b) {
    const __half2 s2 = __half2half2(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sf, __NV_E4M3)));
    uint32_t o[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const uint32_t w = m < 4 ? c.x : c.y;
        const __nv_fp4x2_storage_t pair = (__nv_fp4x2_storage_t)((w >> (8 * (m & 3))) & 0xFFu);
        const __half2 h = __hmul2(__half2(__nv_cvt_fp4x2_to_halfraw2(pair, __NV_E2M1)), s2);
        o[m] = *reinterpret_cast<const uint32_t *>(&h);
    }
    a = make_uint4(o[0], o[1], o[2], o[3]);
    b = make_uint4(o[4], o[5], o[6], o[7]);
}

// 8 f16 -> 8 bf16, for values with at most 8 significant bits (exact).
__device__ __forceinline__ uint4 f16x8_to_bf16x8(uint4 h) {
    uint32_t w[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[m]));
        w[m] = pack_bf2(f.x, f.y);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// ================================================================ reduce

constexpr int kRRows = 32;                 // token rows per reduce pipeline stage
constexpr int kRBox = kRRows * 128;        // [32 rows][64 bf16] = 4 KiB
static_assert(kRRows == 32, "the ReLU pass below maps 128 threads x 4 chunks onto two 32-row boxes");

// F8: k and v are FP8 E4M3 codes; one TMA box per tensor and stage holds the
// 4 heads' 128 codes of 32 tokens (4 KiB), and the MMAs are kind::f8f6f4.
// F4: k and v are NVFP4; a raw stage holds the 4 heads' E2M1 codes of 32
// tokens (2 KiB per tensor, 64 bytes a row) and their E4M3 block scales (a
// 16-byte box per row, of which the group's 8 bytes are used); the transform
// warps decode them into f16 boxes laid out as the bf16 path's tiles (a ring
// of kDec decoded stages, shorter than the raw ring that covers the memory
// latency), and the MMAs are kind::f16 on f16.
template <int IN = kInBf16>
struct RCfg {
    static constexpr bool F8 = IN == kInE4m3, F4 = IN == kInNvfp4;
    // 6 x 8 KiB with FP8 codes, 4 x 16 KiB with bf16, 8 x 5 KiB raw with NVFP4
    static constexpr int kStages = F8 ? 6 : (F4 ? 8 : 4);
    // stage: k boxes, then v boxes
    static constexpr int kVOff = F8 ? kRRows * 128 : 2 * kRBox;
    static constexpr int kStageBytes = F8 ? 2 * kRRows * 128 : (F4 ? 5 * 1024 : kVOff + 2 * kRBox);
    // F4: decoded ring first (1024-byte aligned for the swizzled boxes), then the raw ring
    static constexpr int kDec = F4 ? 3 : 0;
    static constexpr int kDecBytes = 4 * kRBox;
    static constexpr int kRawOff = kDec * kDecBytes;
    static constexpr int kCodeBytes = kRRows * 64;                  // F4: one tensor's codes in a raw stage
    static constexpr int kSfOff = 2 * kCodeBytes;                   // F4: k scales, then v scales (512 B each)
    static constexpr int kRawTx = 2 * kCodeBytes + 2 * kRRows * 16;
    static constexpr int kAuxOff = kRawOff + kStages * kStageBytes; // ones (512 B)
    static constexpr int kAuxBytes = 512;
    static constexpr int kBarOff = kAuxOff + kAuxBytes;
    static constexpr int kNumBars = F4 ? 2 * kStages + 2 * kDec + 1 : 3 * kStages + 1;
    static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
    static constexpr uint32_t kTmemCols = 256;
    // threads that transform the k boxes (warps 2..): NVFP4 8 warps, one
    // 16-feature block of k and one of v per thread and stage; otherwise 4
    // warps, 4 chunks per thread
    static constexpr int kXform = F4 ? 256 : 128;
    static constexpr int kThreadsR = 64 + kXform;
    static_assert(!F4 || kStageBytes >= kRawTx, "the raw stage holds codes and scales");
};

// Fused state combine: the split sums of the CTA's 4 heads ([4][kKVZ] fp32)
// in shared memory, inside the stage ring (no copy or MMA touches the ring
// once the split's last MMA has completed).
constexpr int kFusePartOff = 16384;
constexpr int kZeroRowsOp = kOpRows - kD - 1;   // zero rows 33..47 of the packed operand

// The cluster's share of one head group's combine, in the order of the
// separate combine kernel: S_eff = prior state (with one) + the split sums in
// split order; then the packed bf16 hi + lo operand and (commit) the state.
// The splits of the group are the cluster's CTAs, rank = split.
__device__ void fused_combine(const Plan &p, const Fuse &fz, const float *part, int b, int g, int n, int nthr) {
    const int rank = (int)cluster_ctarank(), P = (int)cluster_nctarank();
    constexpr int kU = 3;   // entries per thread whose remote loads are in flight together
    for (int u0 = rank * nthr + (int)threadIdx.x; u0 < 4 * kKVZ; u0 += kU * P * nthr) {
        float v[kU][kFuseMaxSplits];
#pragma unroll
        for (int j = 0; j < kU; ++j) {
            const int u = u0 + j * P * nthr;
#pragma unroll
            for (int c = 0; c < kFuseMaxSplits; ++c)
                v[j][c] = (c < P && u < 4 * kKVZ) ? ld_dsmem_f32(part + u, (unsigned)c) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kU; ++j) {
            const int u = u0 + j * P * nthr;
            if (u >= 4 * kKVZ) break;
            const int hh = u / kKVZ, e = u - hh * kKVZ;
            const size_t bh = (size_t)b * p.H + 4 * g + hh;
            float run = 0.f;
            if (p.has_state) run = e < kD * kD ? fz.S[bh * kD * kD + e] : fz.Z[bh * kD + e - kD * kD];
#pragma unroll
            for (int c = 0; c < kFuseMaxSplits; ++c)
                if (c < P) run += v[j][c];
            fz.seff[(bh * p.nb + n) * kKVZ + e] = run;
            if (fz.write_bop) {
                const int nrow = e < kD * kD ? (e % kD) : kD;   // value column, or the Z column
                const int kcol = e < kD * kD ? (e / kD) : (e - kD * kD);
                unsigned char *dst = fz.bop + (bh * p.nb + n) * 2 * kOpBytes + op_offset(nrow, kcol);
                const __nv_bfloat16 hi = __float2bfloat16_rn(run);
                *reinterpret_cast<__nv_bfloat16 *>(dst) = hi;
                *reinterpret_cast<__nv_bfloat16 *>(dst + kOpBytes) = __float2bfloat16_rn(run - __bfloat162float(hi));
            }
            if (p.commit) {
                if (e < kD * kD) fz.S[bh * kD * kD + e] = run;
                else fz.Z[bh * kD + e - kD * kD] = run;
            }
        }
    }
    if (fz.write_bop) {
        for (int u = rank * nthr + (int)threadIdx.x; u < 4 * kZeroRowsOp * kD; u += P * nthr) {
            const int hh = u / (kZeroRowsOp * kD), z = u - hh * (kZeroRowsOp * kD);
            const size_t bh = (size_t)b * p.H + 4 * g + hh;
            unsigned char *dst = fz.bop + (bh * p.nb + n) * 2 * kOpBytes + op_offset(kD + 1 + z / kD, z % kD);
            *reinterpret_cast<unsigned short *>(dst) = 0;
            *reinterpret_cast<unsigned short *>(dst + kOpBytes) = 0;
        }
    }
}

// tm_ks, tm_vs: the NVFP4 block scales of k and v (unused otherwise).
template <int IN = kInBf16>
__global__ void __launch_bounds__(RCfg<IN>::kThreadsR, 2)
reduce_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                 float *__restrict__ partials, const Plan p, const Fuse fz) {
    constexpr bool F8 = IN == kInE4m3, F4 = IN == kInNvfp4;
    using C = RCfg<IN>;
    static_assert(kFusePartOff + 4 * kKVZ * 4 <= C::kStages * C::kStageBytes,
                  "the fused split sums fit inside the stages");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *aux = smem + C::kAuxOff;
    // F4: full / raw_free guard the raw ring, relu_done / empty the decoded ring
    constexpr int kRing = F4 ? C::kDec : C::kStages;   // stages the MMAs read
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *relu_done = full + C::kStages;
    uint64_t *empty = relu_done + kRing;
    uint64_t *acc_ready = empty + kRing;
    uint64_t *raw_free = acc_ready + 1;   // F4 only: [kStages], the raw stage has been decoded
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kBarOff + C::kNumBars * 8);
    volatile int *abort_word = reinterpret_cast<volatile int *>(tmem_slot + 1);

    // the splits of a head group are consecutive CTAs (one cluster when fused)
    const int G = p.H / 4;
    long long id = blockIdx.x;
    const int sp = (int)(id % p.P); id /= p.P;
    const int g = (int)(id % G); id /= G;
    const int n = (int)(id % p.nb); id /= p.nb;
    const int b = (int)id;
    const long long blk0 = (long long)n * p.L;
    const long long blk1 = blk0 + p.L < p.N ? blk0 + p.L : (long long)p.N;
    const long long t0 = blk0 + (long long)sp * p.chunk;
    const long long t1 = t0 + p.chunk < blk1 ? t0 + p.chunk : blk1;
    const int nst = t1 > t0 ? (int)((t1 - t0 + kRRows - 1) / kRRows) : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *fpart = reinterpret_cast<float *>(smem + kFusePartOff);

    // k, v (and the prior state) may come from the kernel just before this one:
    // wait for it, then let the next kernel be scheduled
    pdl_wait();
    pdl_trigger();

    if (nst == 0 && fz.on) {   // a split past the end of a short block: zero sums, still in the cluster
        for (int e = threadIdx.x; e < 4 * kKVZ; e += C::kThreadsR) fpart[e] = 0.f;
        __syncthreads();
        cluster_sync();
        fused_combine(p, fz, fpart, b, g, n, C::kThreadsR);
        cluster_sync();
        return;
    }
    if (nst == 0) {   // a split past the end of a short last block: its sums are zero
        for (int e = threadIdx.x; e < 4 * kKVZ; e += C::kThreadsR) {
            const int h = g * 4 + e / kKVZ;
            partials[((((size_t)b * p.H + h) * p.nb + n) * p.P + sp) * kKVZ + e % kKVZ] = 0.f;
        }
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) mbar_init(&full[s], 1);
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&relu_done[s], C::kXform);
            mbar_init(&empty[s], 1);
        }
        if constexpr (F4)
            for (int s = 0; s < C::kStages; ++s) mbar_init(&raw_free[s], C::kXform);
        mbar_init(acc_ready, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    // B operand of the z contraction: 16 x 16 ones (any layout reads 1.0)
    // (1.0 is 0x3F80 in bf16, 0x38 in E4M3, 0x3C00 in f16)
    for (int i = threadIdx.x; i < 128; i += C::kThreadsR)
        reinterpret_cast<uint32_t *>(aux)[i] = F8 ? 0x38383838u : (F4 ? 0x3C003C00u : 0x3F803F80u);
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        if constexpr (F4) {
            prefetch_tmap(&tm_ks);
            prefetch_tmap(&tm_vs);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0;

    if (warp == kWarpTma) {
        if (lane == 0) {
            const int c0 = g * 128;   // first feature of the group (a code = a byte with F8)
            for (int i = 0; i < nst; ++i) {
                const int s = i % C::kStages;
                const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
                if (!mbar_wait(F4 ? &raw_free[s] : &empty[s], ph ^ 1u, abort_word, &g_wait_flag, 1)) break;
                uint8_t *st = smem + C::kRawOff + s * C::kStageBytes;
                const int row = (int)(t0 + (long long)kRRows * i);
                if constexpr (F4) {
                    // codes: the group's 4 x 16 bytes of a row; scales: the 16-byte
                    // aligned box holding the group's 8 bytes
                    mbar_arrive_expect_tx(&full[s], C::kRawTx);
                    tma_load_3d(st, &tm_k, &full[s], g * 64, row, b);
                    tma_load_3d(st + C::kCodeBytes, &tm_v, &full[s], g * 64, row, b);
                    tma_load_3d(st + C::kSfOff, &tm_ks, &full[s], (g >> 1) * 16, row, b);
                    tma_load_3d(st + C::kSfOff + kRRows * 16, &tm_vs, &full[s], (g >> 1) * 16, row, b);
                } else if constexpr (F8) {
                    mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                    tma_load_3d(st, &tm_k, &full[s], c0, row, b);
                    tma_load_3d(st + C::kVOff, &tm_v, &full[s], c0, row, b);
                } else {
                    mbar_arrive_expect_tx(&full[s], 4 * kRBox);
                    tma_load_3d(st, &tm_k, &full[s], c0, row, b);
                    tma_load_3d(st + kRBox, &tm_k, &full[s], c0 + 64, row, b);
                    tma_load_3d(st + C::kVOff, &tm_v, &full[s], c0, row, b);
                    tma_load_3d(st + C::kVOff + kRBox, &tm_v, &full[s], c0 + 64, row, b);
                }
                issued = i + 1;
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t id_kv = F8 ? idesc_e4m3(128, 128, 1, 1) : (F4 ? idesc_f16(128, 128, 1, 1) : idesc_bf16(128, 128, 1, 1));
            const uint32_t id_z = F8 ? idesc_e4m3(128, 16, 1, 0) : (F4 ? idesc_f16(128, 16, 1, 0) : idesc_bf16(128, 16, 1, 0));
            // ones: K-major, no swizzle, 32 bytes of K per row either way
            const uint64_t d_ones = smem_desc(smem_u32(aux), 128, 256, kLayoutNone);
            for (int i = 0; i < nst; ++i) {
                const int s = i % kRing;
                const uint32_t ph = (uint32_t)(i / kRing) & 1u;
                if (!mbar_wait(&relu_done[s], ph, abort_word, &g_wait_flag, 2)) break;
                tc_fence_after();
                const uint32_t kaddr = smem_u32(smem + s * (F4 ? C::kDecBytes : C::kStageBytes));
                const uint32_t vaddr = kaddr + C::kVOff;
                if constexpr (F8) {
                    // MN-major, 128-byte swizzle: the 128 codes of a token are one
                    // 128-byte row; K = 32 tokens = four 8-row groups 1024 B apart
                    const uint64_t da = smem_desc(kaddr, 4096, 1024, kLayoutSw128);
                    const uint64_t db = smem_desc(vaddr, 4096, 1024, kLayoutSw128);
                    const uint32_t acc = i > 0 ? 1u : 0u;
                    mma_f8(tmem, da, db, id_kv, acc);
                    mma_f8(tmem + 128, da, d_ones, id_z, acc);
                    mma_commit(&empty[s]);
                    continue;
                }
#pragma unroll
                for (int kk = 0; kk < kRRows / 16; ++kk) {
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
        const int wt = threadIdx.x - 64;   // 0 .. C::kXform - 1

        for (int i = 0; i < nst; ++i) {
            const int s = i % C::kStages;
            const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
            if (!mbar_wait(&full[s], ph, abort_word, &g_wait_flag, 3)) break;
            const int ds = F4 ? i % kRing : s;   // the stage the MMAs read
            uint8_t *kt = smem + (F4 ? ds * C::kDecBytes : s * C::kStageBytes);
            const long long row0 = t0 + (long long)kRRows * i;
            if constexpr (F4) {
                // the decoded stage is free once the MMAs of stage i - kDec are done
                if (!mbar_wait(&empty[ds], ((uint32_t)(i / kRing) & 1u) ^ 1u, abort_word, &g_wait_flag, 5)) break;
                const uint8_t *raw = smem + C::kRawOff + s * C::kStageBytes;
                // this thread: block u of k and of v, u = (row, head, 16-feature half)
                const int u = wt;
                const int r = u >> 3, hd = (u >> 1) & 3, fb = u & 1;
                const int L0 = (hd & 1) * 4 + fb * 2;   // logical chunks L0, L0 + 1 of box hd / 2
                uint8_t *drow = kt + (hd >> 1) * kRBox + r * 128;
                const int p0 = (L0 ^ (r & 7)) << 4, p1 = ((L0 + 1) ^ (r & 7)) << 4;
                const int cb = r * 64 + hd * 16 + fb * 8;                        // code bytes in the raw boxes
                const int sb = C::kSfOff + r * 16 + (g & 1) * 8 + hd * 2 + fb;   // scale byte
                uint2 ck = *reinterpret_cast<const uint2 *>(raw + cb);
                const uint2 cv = *reinterpret_cast<const uint2 *>(raw + C::kCodeBytes + cb);
                const uint8_t sk = raw[sb], sv = raw[sb + kRRows * 16];
                if (row0 + r < t1) {
                    ck.x = relu_e2m1x8(ck.x);
                    ck.y = relu_e2m1x8(ck.y);
                } else {
                    ck = make_uint2(0u, 0u);   // rows past the split contribute nothing
                }
                // The 8 lanes of a shared-memory phase are one row: heads 0, 1
                // write box 0 and heads 2, 3 box 1, 4 KiB apart, so the same
                // chunk of both boxes falls on the same banks.  The box-1 lanes
                // store their two chunks in the other order, so that every phase
                // writes 8 distinct chunk positions (one wavefront, not two).
                const bool swap = (hd >> 1) != 0;
                const int pa = swap ? p1 : p0, pb = swap ? p0 : p1;
                uint4 a, bq;
                decode_nvfp4_16(ck, sk, a, bq);
                *reinterpret_cast<uint4 *>(drow + pa) = swap ? bq : a;
                *reinterpret_cast<uint4 *>(drow + pb) = swap ? a : bq;
                decode_nvfp4_16(cv, sv, a, bq);
                *reinterpret_cast<uint4 *>(drow + C::kVOff + pa) = swap ? bq : a;
                *reinterpret_cast<uint4 *>(drow + C::kVOff + pb) = swap ? a : bq;
            } else if constexpr (F8) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {             // the k box: 256 chunks of 16 codes, 2 per thread
                    const int c = wt + 128 * j;
                    const int r = c >> 3;                 // token row (8 chunks of 16 B per 128-byte row)
                    uint4 *ptr = reinterpret_cast<uint4 *>(kt + (size_t)c * 16);
                    uint4 x = *ptr;
                    if (row0 + r < t1) {
                        // E4M3 codes as signed bytes: every negative value (sign bit
                        // set, -0 included) is below 0, so a signed max with 0 is ReLU
                        x.x = __vmaxs4(x.x, 0u); x.y = __vmaxs4(x.y, 0u);
                        x.z = __vmaxs4(x.z, 0u); x.w = __vmaxs4(x.w, 0u);
                    } else {
                        x = make_uint4(0u, 0u, 0u, 0u);   // rows past the split contribute nothing
                    }
                    *ptr = x;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) {             // 512 chunks of 16 bytes: 4 per thread
                    const int c = wt + 128 * j;           // 16-byte chunk of the two k boxes
                    const int r = (c % (8 * kRRows)) >> 3;   // token row inside its box
                    uint4 *ptr = reinterpret_cast<uint4 *>(kt + (size_t)c * 16);
                    uint4 x = *ptr;
                    if (row0 + r < t1) {
                        x.x = relu2(x.x); x.y = relu2(x.y); x.z = relu2(x.z); x.w = relu2(x.w);
                    } else {
                        x = make_uint4(0u, 0u, 0u, 0u);   // rows past the split contribute nothing
                    }
                    *ptr = x;
                }
            }
            // the generic reads and writes of this stage before the tensor cores
            // read the decoded boxes and TMA refills the raw stage (async proxy)
            fence_proxy_async_smem();
            if constexpr (F4) mbar_arrive(&raw_free[s]);
            mbar_arrive(&relu_done[ds]);
        }
        // epilogue: warp quarter q reads TMEM lanes 32q.. = key features of head 4g+q.
        // Every work thread reaches the named barrier, and the TMEM read is
        // taken or skipped by whole warps, even after a wait gave up.
        bool got = mbar_wait(acc_ready, 0, abort_word, &g_wait_flag, 4);
        got = __all_sync(0xffffffffu, got);
        const int qd = warp & 3;
        const int h = g * 4 + qd;
        float z = 0.f;
        // warps 2..5 (one per TMEM lane quarter) write the split sums
        if (got && warp < 6) {
            tc_fence_after();
            const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
            float kv[32];
            tmem_ld32(tmem + lane_off + 32 * qd, kv);
            z = tmem_ld1(tmem + lane_off + 128);
            tmem_wait_ld();
            if constexpr (F8 || F4) {
                // per-tensor scales: KV = sk sv sum phi(k^) v^T, z = sk sum phi(k^)
                const float skv = p.sk * p.sv;
#pragma unroll
                for (int j = 0; j < 32; ++j) kv[j] *= skv;
                z *= p.sk;
            }
            float *dst = fz.on ? fpart + qd * kKVZ : partials + ((((size_t)b * p.H + h) * p.nb + n) * p.P + sp) * kKVZ;
            float4 *drow = reinterpret_cast<float4 *>(dst + lane * kD);
#pragma unroll
            for (int j = 0; j < 8; ++j) drow[j] = make_float4(kv[4 * j], kv[4 * j + 1], kv[4 * j + 2], kv[4 * j + 3]);
            dst[kD * kD + lane] = z;
        }
    }

    // teardown: nothing may still write this CTA's shared memory or TMEM
    if (warp == kWarpTma && lane == 0 && *abort_word) {
        for (int i = issued - C::kStages < 0 ? 0 : issued - C::kStages; i < issued; ++i)
            final_wait(&full[i % C::kStages], (uint32_t)(i / C::kStages) & 1u);
    }
    if (warp == kWarpMma && lane == 0) final_wait(acc_ready, 0);
    tc_fence_before();
    // lanes that skipped the single-lane roles wait for their lane 0 here, so
    // every warp reaches the block barrier whole
    __syncwarp();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if (fz.on) {   // every split's sums are in its CTA's shared memory: combine them
        cluster_sync();
        fused_combine(p, fz, fpart, b, g, n, C::kThreadsR);
        cluster_sync();   // no CTA leaves while another still reads its shared memory
    }
}

// ================================================================ apply

constexpr int kATile = 128 * 128;              // [128 rows][64 bf16] = 16 KiB: 2 heads
constexpr int kABopBytes = 2 * 2 * kOpBytes;   // 2 heads x (hi, lo)
constexpr int kAThreads = 320;                 // 10 warps
constexpr int kAXform0 = 192;                  // first thread of the transform warps 6..9
constexpr int kAWarpStg = 32 * 128;            // one epilogue warp's staging box: [32 rows][64 bf16]

template <int IN = kInBf16>
struct ACfg {
    static constexpr bool F8 = IN == kInE4m3, F4 = IN == kInNvfp4;
    // F8: a stage is the bf16 tile the MMA reads (16 KiB, 128-byte swizzle)
    // followed by the tile's E4M3 codes as TMA lands them (8 KiB, no swizzle).
    // F4: the bf16 tile, the tile's E2M1 codes (4 KiB: 32 bytes a row) and
    // the 16-byte box of E4M3 block scales of each row (2 KiB)
    static constexpr int kStages = (F8 || F4) ? 3 : 4;
    static constexpr int kCodeOff = kATile;
    static constexpr int kSfOff = kATile + kATile / 4;   // F4
    static constexpr int kQTx = F8 ? kATile / 2 : (F4 ? kATile / 4 + 128 * 16 : kATile);   // bytes TMA lands per tile
    static constexpr int kStageBytes = F8 ? kATile + kATile / 2 : (F4 ? kSfOff + 128 * 16 : kATile);
    static constexpr int kStgBufs = F8 ? 1 : 2;                        // staging boxes per epilogue warp
    static constexpr int kOutOff = kStages * kStageBytes;
    static constexpr int kBopOff = kOutOff + 4 * kStgBufs * kAWarpStg;
    static constexpr int kBarOff = kBopOff + kABopBytes;
    static constexpr int kNumBars = 3 * kStages + 2 + 2 + 3;          // + acc[2], acc_empty[2], bop, drain, dep
    static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
    static constexpr int kAccCols = 96;                                // per TMEM buffer (2 heads)
    static constexpr int kHeadCols = kOpRows;
    static constexpr uint32_t kTmemCols = 256;
};

// Warp roles: 0 issues TMA, 1 owns TMEM and issues the MMAs, 2..5 run the
// epilogue (warp w reads TMEM lanes 32*(w%4).. = token rows of the tile),
// 6..9 apply phi to the q tiles in shared memory.  The transform
// of tile i+1 and the epilogue of tile i run at the same time.
// tm_qs: the NVFP4 block scales of q (unused otherwise).
template <int IN = kInBf16>
__global__ void __launch_bounds__(kAThreads, 2)
apply_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qs,
                const __grid_constant__ CUtensorMap tm_out, __nv_bfloat16 *__restrict__ out,
                const uint8_t *__restrict__ bop, const float *__restrict__ seff, const Plan p) {
    constexpr bool F8 = IN == kInE4m3, F4 = IN == kInNvfp4;
    using C = ACfg<IN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stg = smem + C::kOutOff;
    uint8_t *bops = smem + C::kBopOff;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *xform_done = full + C::kStages;
    uint64_t *empty = xform_done + C::kStages;
    uint64_t *acc_full = empty + C::kStages;   // [2]
    uint64_t *acc_empty = acc_full + 2;        // [2]
    uint64_t *bop_full = acc_empty + 2;
    uint64_t *drain = bop_full + 1;            // only used when a wait gave up
    uint64_t *dep_ready = drain + 1;           // the previous kernel (state combine) has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dep_ready + 1);
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
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xform_done[s], kWork);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kWork);
        }
        mbar_init(bop_full, 1);
        mbar_init(drain, 1);
        mbar_init(dep_ready, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_out);
        if constexpr (F4) prefetch_tmap(&tm_qs);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0;
    bool bop_issued = false;

    if (warp == kWarpTma) {
        if (lane == 0) {
            auto load_q = [&](int i, int s) {
                uint8_t *st = smem + s * C::kStageBytes;
                const int row = (int)(ta0 + 128LL * i);
                mbar_arrive_expect_tx(&full[s], C::kQTx);
                if constexpr (F4) {
                    // the pair's 2 x 16 code bytes; the 16-byte aligned box holding its 4 scale bytes
                    tma_load_3d(st + C::kCodeOff, &tm_q, &full[s], hp * 32, row, b);
                    tma_load_3d(st + C::kSfOff, &tm_qs, &full[s], (hp >> 2) * 16, row, b);
                } else {
                    tma_load_3d(st + (F8 ? C::kCodeOff : 0), &tm_q, &full[s], hp * 64, row, b);
                }
                issued = i + 1;
            };
            // q is an input of the call, complete before the reduce of this call
            // started: its first tiles are fetched while the state combine still runs
            const int pre = ntiles < C::kStages ? ntiles : C::kStages;
            for (int i = 0; i < pre; ++i) load_q(i, i);
            pdl_wait();   // the packed operand and Z_eff are written by the previous kernel
            mbar_arrive(dep_ready);
            mbar_arrive_expect_tx(bop_full, kABopBytes);
            for (int hh = 0; hh < 2; ++hh) {
                const size_t src = (((size_t)b * p.H + 2 * hp + hh) * p.nb + n) * 2 * kOpBytes;
                bulk_load(bops + hh * 2 * kOpBytes, bop + src, 2 * kOpBytes, bop_full);
            }
            bop_issued = true;
            for (int i = pre; i < ntiles; ++i) {
                const int s = i % C::kStages;
                const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, &g_wait_flag, 11)) break;
                load_q(i, s);
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, C::kHeadCols, 0, 0);
            const uint32_t baddr = smem_u32(bops);
            if (mbar_wait(bop_full, 0, abort_word, &g_wait_flag, 12)) {
                for (int i = 0; i < ntiles; ++i) {
                    const int s = i % C::kStages;
                    const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
                    const int ab = i & 1;
                    const uint32_t aph = (uint32_t)(i >> 1) & 1u;
                    if (!mbar_wait(&xform_done[s], ph, abort_word, &g_wait_flag, 13)) break;
                    if (!mbar_wait(&acc_empty[ab], aph ^ 1u, abort_word, &g_wait_flag, 14)) break;
                    tc_fence_after();
                    const uint32_t qaddr = smem_u32(smem + s * C::kStageBytes);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t d = tmem + ab * C::kAccCols + hh * C::kHeadCols;
                        // (A part, B part) products: hi.hi, hi.lo
#pragma unroll
                        for (int prod = 0; prod < 2; ++prod) {
                            const int apart = prod == 2 ? 1 : 0;
                            const int bpart = prod == 1 ? 1 : 0;
#pragma unroll
                            for (int kk = 0; kk < 2; ++kk) {
                                // A: K-major, 128-byte swizzle; head hh is the 64-byte half
                                // of each 128-byte row, 16 features = 32 bytes per step
                                const uint64_t da = smem_desc(qaddr + apart * kATile + hh * 64 + kk * 32, 16, 1024,
                                                              kLayoutSw128);
                                // B: K-major, no swizzle, core matrices 128 B apart along K,
                                // 8-row groups 512 B apart; 16 features = 256 bytes per step
                                const uint64_t db = smem_desc(baddr + hh * 2 * kOpBytes + bpart * kOpBytes + kk * 256,
                                                              128, 512, kLayoutNone);
                                mma_bf16(d, da, db, idesc, (prod | kk) ? 1u : 0u);
                            }
                        }
                    }
                    mma_commit(&empty[s]);
                    mma_commit(&acc_full[ab]);
                }
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------ transform warps
        const int tt = threadIdx.x - kAXform0;   // 0..127
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % C::kStages;
            const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
            if (ok && !mbar_wait(&full[s], ph, abort_word, &g_wait_flag, 15)) ok = false;
            uint8_t *qt = smem + s * C::kStageBytes;
            const long long row0 = ta0 + 128LL * i;
            if (F4 && ok) {
                // NVFP4 [128 rows][2 heads][32 codes] -> phi(q) in bf16, exact (<= 6
                // significant bits), into the 128-byte swizzled tile the MMA reads:
                // 4 blocks of 16 features per thread
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int u = tt + 128 * j;
                    const int rr = u >> 2, hd = (u >> 1) & 1, fb = u & 1;
                    uint2 c = *reinterpret_cast<const uint2 *>(qt + C::kCodeOff + rr * 32 + hd * 16 + fb * 8);
                    const uint8_t sf = qt[C::kSfOff + rr * 16 + (hp & 3) * 4 + hd * 2 + fb];
                    c.x = relu_e2m1x8(c.x);
                    c.y = relu_e2m1x8(c.y);
                    uint4 a, bq;
                    decode_nvfp4_16(c, sf, a, bq);
                    const int L0 = hd * 4 + fb * 2;
                    *reinterpret_cast<uint4 *>(qt + rr * 128 + ((L0 ^ (rr & 7)) << 4)) = f16x8_to_bf16x8(a);
                    *reinterpret_cast<uint4 *>(qt + rr * 128 + (((L0 + 1) ^ (rr & 7)) << 4)) = f16x8_to_bf16x8(bq);
                }
            } else if (F8 && ok) {
                // E4M3 codes [128 rows][64] -> phi(q) in bf16, exact (<= 4 significant
                // bits), into the 128-byte swizzled tile the MMA reads
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int u = tt + 128 * j;
                    const int rr = u >> 3, L = u & 7;       // token row, logical chunk of 8 features
                    const uint2 c8 = *reinterpret_cast<const uint2 *>(qt + C::kCodeOff + rr * 64 + L * 8);
                    const uint32_t w[2] = {__vmaxs4(c8.x, 0u), __vmaxs4(c8.y, 0u)};   // ReLU on the codes
                    uint32_t o[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)(w[m >> 1] >> (16 * (m & 1)));
                        const __half2 hv = __half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3));
                        const float2 fv = __half22float2(hv);
                        o[m] = pack_bf2(fv.x, fv.y);
                    }
                    *reinterpret_cast<uint4 *>(qt + rr * 128 + ((L ^ (rr & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            } else if (ok) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 *ptr = reinterpret_cast<uint4 *>(qt + (size_t)(tt + 128 * j) * 16);
                    uint4 x = *ptr;
                    x.x = relu2(x.x); x.y = relu2(x.y); x.z = relu2(x.z); x.w = relu2(x.w);
                    *ptr = x;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&xform_done[s]);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int qd = warp & 3;
        const int r = 32 * qd + lane;               // token row of this thread in a tile
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        uint8_t *wstg = stg + qd * C::kStgBufs * kAWarpStg;   // this warp's staging boxes
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int ab = i & 1;
            const uint32_t aph = (uint32_t)(i >> 1) & 1u;
            bool got = ok && mbar_wait(&acc_full[ab], aph, abort_word, &g_wait_flag, 16);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
            float num0[32], num1[32], den0 = 0.f, den1 = 0.f;
            if (got) {
                tc_fence_after();
                const uint32_t base = tmem + lane_off + ab * C::kAccCols;
                tmem_ld32(base, num0);
                tmem_ld32(base + C::kHeadCols, num1);
                den0 = tmem_ld1(base + kD);
                den1 = tmem_ld1(base + C::kHeadCols + kD);
                tmem_wait_ld();
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);

            const long long row0 = ta0 + 128LL * i;
            const long long wrow0 = row0 + 32 * qd;    // first row of this warp
            // TMA store of the warp's 32 rows unless they run into another block
            // (rows past the end of the tensor are clipped by TMA)
            const bool boxed = wrow0 + 32 <= ta1 || ta1 == p.N;
            if (boxed) {
                uint8_t *sb = wstg + (i % C::kStgBufs) * kAWarpStg;
                if (lane == 0) bulk_wait_read<C::kStgBufs - 1>();   // the last store from sb has read it
                __syncwarp();
                if (got) {
                    // F8, F4: out = sq num^ / (sq den^ + eps) with num^, den^ from the codes
                    const float qs = (F8 || F4) ? p.sq : 1.0f;
                    const float inv0 = qs / (qs * den0 + p.eps), inv1 = qs / (qs * den1 + p.eps);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {       // logical 16-byte chunk c: head c/4
                        const float *v = c < 4 ? num0 : num1;
                        const float inv = c < 4 ? inv0 : inv1;
                        const int f0 = 8 * (c & 3);
                        const int pc = c ^ (lane & 7);  // 128-byte swizzle (row % 8 == lane % 8)
                        *reinterpret_cast<uint4 *>(sb + lane * 128 + pc * 16) =
                            make_uint4(pack_bf2(v[f0] * inv, v[f0 + 1] * inv), pack_bf2(v[f0 + 2] * inv, v[f0 + 3] * inv),
                                       pack_bf2(v[f0 + 4] * inv, v[f0 + 5] * inv), pack_bf2(v[f0 + 6] * inv, v[f0 + 7] * inv));
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && ok) {
                    tma_store_3d(&tm_out, sb, hp * 64, (int)wrow0, b);
                    bulk_commit();
                }
            } else if (got && row0 + r < ta1) {
                // a short last tile inside the tensor: the rows after ta1 belong to another block
                const float qs = (F8 || F4) ? p.sq : 1.0f;
                const float inv0 = qs / (qs * den0 + p.eps), inv1 = qs / (qs * den1 + p.eps);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float *v = hh ? num1 : num0;
                    const float inv = hh ? inv1 : inv0;
                    uint4 *dst = reinterpret_cast<uint4 *>(out + (((size_t)b * p.N + row0 + r) * p.H + 2 * hp + hh) * kD);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        dst[c] = make_uint4(pack_bf2(v[8 * c] * inv, v[8 * c + 1] * inv),
                                            pack_bf2(v[8 * c + 2] * inv, v[8 * c + 3] * inv),
                                            pack_bf2(v[8 * c + 4] * inv, v[8 * c + 5] * inv),
                                            pack_bf2(v[8 * c + 6] * inv, v[8 * c + 7] * inv));
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    if (warp == kWarpTma && lane == 0 && *abort_word) {
        if (bop_issued) final_wait(bop_full, 0);
        for (int i = issued - C::kStages < 0 ? 0 : issued - C::kStages; i < issued; ++i)
            final_wait(&full[i % C::kStages], (uint32_t)(i / C::kStages) & 1u);
    }
    if (warp == kWarpMma && lane == 0 && *abort_word) {
        // make every MMA issued so far finish before TMEM is released
        mma_commit(drain);
        final_wait(drain, 0);
    }
    tc_fence_before();
    // lanes that skipped the single-lane roles wait for their lane 0 here, so
    // every warp reaches the block barrier whole
    __syncwarp();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
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

// 3D view of a [B][N][row_bytes] tensor of bytes (E4M3 codes: H*32 bytes a
// row; NVFP4 codes: H*16; NVFP4 block scales: H*2): boxes of box_inner bytes
// x box_rows tokens, 128-byte swizzle or none.
bool make_map_bytes(CUtensorMap *m, const void *base, int B, int N, long long row_bytes, int box_inner,
                    int box_rows, bool sw128) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * (cuuint64_t)N};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool smem_ready() {
    static std::once_flag once;
    static bool ok = false;
    std::call_once(once, [] {
        ok = set_smem((const void *)reduce_tc_kernel<kInBf16>, RCfg<kInBf16>::kSmem) &&
             set_smem((const void *)apply_tc_kernel<kInBf16>, ACfg<kInBf16>::kSmem) &&
             set_smem((const void *)reduce_tc_kernel<kInE4m3>, RCfg<kInE4m3>::kSmem) &&
             set_smem((const void *)apply_tc_kernel<kInE4m3>, ACfg<kInE4m3>::kSmem) &&
             set_smem((const void *)reduce_tc_kernel<kInNvfp4>, RCfg<kInNvfp4>::kSmem) &&
             set_smem((const void *)apply_tc_kernel<kInNvfp4>, ACfg<kInNvfp4>::kSmem);
    });
    return ok;
}

}  // namespace

bool tc_available() {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
    return major == 10 && minor == 0 && encode_fn() != nullptr;
}

bool make_bf16_map(CUtensorMap *m, const void *base, int B, int N, int H, int box_rows) {
    return make_map(m, base, B, N, H, box_rows);
}

bool make_u8_map(CUtensorMap *m, const void *base, int B, int N, long long row_bytes, int box_inner, int box_rows,
                 int swizzle_bytes) {
    auto fn = encode_fn();
    if (!fn || (swizzle_bytes != 0 && swizzle_bytes != 64 && swizzle_bytes != 128)) return false;
    cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * (cuuint64_t)N};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                        : CU_TENSOR_MAP_SWIZZLE_NONE;
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_bf16_map_nd(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                      const cuuint64_t *strides, const cuuint32_t *box) {
    auto fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


int launch_reduce_tc(const void *k, const void *v, float *partials, const Plan &p, cudaStream_t s, const Fuse *fz) {
    if (p.rope || !smem_ready()) return -1;   // RoPE calls take the kernels of k_rope_tc.cu
    CUtensorMap mk, mv, mks{}, mvs{};
    const long long grid = (long long)p.B * (p.H / 4) * p.nb * p.P;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    const Fuse off = {nullptr, nullptr, nullptr, nullptr, 0, 0};
    const Fuse f = fz ? *fz : off;
    if (f.on && (p.nb != 1 || p.P < 1 || p.P > kFuseMaxSplits)) return -1;
    auto go = [&](auto kernel, int threads, int smem) {
        return f.on ? launch_pdl_cluster(kernel, (unsigned)grid, threads, smem, (unsigned)p.P, s, mk, mv, mks, mvs,
                                         partials, p, f)
                    : launch_pdl(kernel, (unsigned)grid, threads, smem, s, mk, mv, mks, mvs, partials, p, f);
    };
    if (p.f4) {
        // codes: the group's 64 bytes of a row; scales: 16-byte boxes (H % 8 == 0)
        if (p.H % 8 != 0 || !make_map_bytes(&mk, k, p.B, p.N, (long long)p.H * kD / 2, 64, kRRows, false) ||
            !make_map_bytes(&mv, v, p.B, p.N, (long long)p.H * kD / 2, 64, kRRows, false) ||
            !make_map_bytes(&mks, p.sfk, p.B, p.N, (long long)p.H * kD / 16, 16, kRRows, false) ||
            !make_map_bytes(&mvs, p.sfv, p.B, p.N, (long long)p.H * kD / 16, 16, kRRows, false))
            return -1;
        using C4 = RCfg<kInNvfp4>;
        return go(reduce_tc_kernel<kInNvfp4>, C4::kThreadsR, C4::kSmem) ? 1 : -1;
    }
    if (p.f8) {
        if (!make_map_bytes(&mk, k, p.B, p.N, (long long)p.H * kD, 128, kRRows, true) ||
            !make_map_bytes(&mv, v, p.B, p.N, (long long)p.H * kD, 128, kRRows, true))
            return -1;
        using C8 = RCfg<kInE4m3>;
        return go(reduce_tc_kernel<kInE4m3>, C8::kThreadsR, C8::kSmem) ? 1 : -1;
    }
    if (!make_map(&mk, k, p.B, p.N, p.H, kRRows) || !make_map(&mv, v, p.B, p.N, p.H, kRRows)) return -1;
    return go(reduce_tc_kernel<kInBf16>, RCfg<kInBf16>::kThreadsR, RCfg<kInBf16>::kSmem) ? 1 : -1;
}

int launch_apply_tc(const void *q, void *out, const void *bop, const float *seff, const Plan &p, cudaStream_t s) {
    if (p.rope || !smem_ready()) return -1;   // RoPE calls take the kernels of k_rope_tc.cu
    CUtensorMap mq, mqs{}, mo;
    const long long grid = (long long)p.B * p.nb * p.Pa * (p.H / 2);
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
    const uint8_t *bb = static_cast<const uint8_t *>(bop);
    if (!make_map(&mo, out, p.B, p.N, p.H, 32)) return -1;
    if (p.f4) {
        // q codes: the pair's 32 bytes x 128 tokens; scales: 16-byte boxes (H % 8 == 0)
        if (p.H % 8 != 0 || !make_map_bytes(&mq, q, p.B, p.N, (long long)p.H * kD / 2, 32, 128, false) ||
            !make_map_bytes(&mqs, p.sfq, p.B, p.N, (long long)p.H * kD / 16, 16, 128, false))
            return -1;
        return launch_pdl(apply_tc_kernel<kInNvfp4>, (unsigned)grid, kAThreads, ACfg<kInNvfp4>::kSmem,
                          s, mq, mqs, mo, o, bb, seff, p)
                   ? 1
                   : -1;
    }
    if (p.f8) {
        // q codes: boxes of the 2 heads' 64 codes x 128 tokens, no swizzle; out bf16
        if (!make_map_bytes(&mq, q, p.B, p.N, (long long)p.H * kD, 64, 128, false)) return -1;
        return launch_pdl(apply_tc_kernel<kInE4m3>, (unsigned)grid, kAThreads, ACfg<kInE4m3>::kSmem,
                          s, mq, mqs, mo, o, bb, seff, p)
                   ? 1
                   : -1;
    }
    if (!make_map(&mq, q, p.B, p.N, p.H, 128)) return -1;
    return launch_pdl(apply_tc_kernel<kInBf16>, (unsigned)grid, kAThreads, ACfg<kInBf16>::kSmem, s, mq, mqs, mo, o, bb,
                      seff, p)
               ? 1
               : -1;
}

namespace {
// One CTA waits on an mbarrier that nothing arrives at: the bounded wait gives
// up after its time limit, raises the device flag and the kernel returns.
__global__ void bounded_wait_selftest_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_word;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_word = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_word, &g_wait_flag, 99);
}
}  // namespace

int launch_bounded_wait_selftest(cudaStream_t s) {
    bounded_wait_selftest_kernel<<<1, 32, 0, s>>>();
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int read_and_clear_device_flag(cudaStream_t s, unsigned *flag_out) {
    unsigned zero = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(flag_out, g_wait_flag, sizeof(unsigned)) != cudaSuccess) return -1;
    if (*flag_out && cudaMemcpyToSymbol(g_wait_flag, &zero, sizeof(unsigned)) != cudaSuccess) return -1;
    return 0;
}

}  // namespace la
