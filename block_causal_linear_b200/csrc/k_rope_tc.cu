// k_rope_tc.cu -- tensor-core reduce and apply for bf16 inputs with 3D RoPE on
// phi(q), phi(k) in the numerator (sd114.wiki SANA-Video summary, section
// "两大核心技术突破", item 1: the kernel feature map, with RoPE for the
// spatio-temporal position of each latent token).
//
// reduce: per (b, 4-head group, block) KV_n = sum_t R phi(k_t)^T v_t and
//   z_n = sum_t phi(k_t), the block's KV product that is then added to the
//   cumulative state ("Nvidia, MIT ve diğerleri video yapay zeka devrimini
//   başlattı", section "Sabit Bellekli KV önbelleğe alma mekanizması").
//   Per 16 tokens one M=128 x N=128 x K=16 MMA per part: A = R phi(K) of the
//   4 heads (MN-major, 128-byte swizzle), B = V of the same heads straight
//   from the TMA tile; only the 4 diagonal 32x32 blocks of D are used.  The
//   rotated features go to the tensor cores as a bf16 hi and a lo part
//   (R phi(k) = hi + lo to about 16 bits), fp32 accumulation in TMEM; z is
//   summed on the CUDA cores from the unrotated phi(k).
// apply: out_t = R phi(q_t) S_eff / (phi(q_t) . Z_eff + eps) per 128-token
//   tile of 2 heads: the numerator as (R phi(q))_hi S_hi + (R phi(q))_hi S_lo
//   + (R phi(q))_lo S_hi (N = 32) with S_eff the combine's packed bf16 hi + lo
//   operand, the unrotated denominator summed in fp32 on the CUDA cores while
//   the tile is transformed; the epilogue divides, rounds to bf16 and stores
//   with TMA.
//
// Both kernels run one CTA per SM over a stream-K plan (la_internal.cuh, Sk):
// the call's work in (b, block, unit) order is cut into equal contiguous
// ranges, so that every SM gets the same share whatever B, H and the block
// length are.  A reduce CTA writes one set of split sums per unit it meets
// into slot (its index - the index of the unit's first CTA); the combine
// kernel adds a unit's slots in CTA order, so results are bitwise
// reproducible.
//
// Shared memory is laid out for depth: the TMA tiles land in a ring of raw
// stages (160 KiB in the reduce, 176 KiB in the apply) separate from the
// transformed operands the tensor cores read (shared memory in the reduce,
// tensor memory in the apply), so that a raw stage is free as soon as the
// transform has read it.  The cos/sin table holds records of
// two feature pairs (cos a, cos b, sin a, sin b) per position of each axis;
// a transform thread owns one token row, so the 8 lanes of a shared-memory
// phase read 8 consecutive rows: distinct 16-byte chunks of the swizzled
// tiles, and for the column axis distinct consecutive records.
//
// Warp roles (736 threads): 0 and 6 TMA (even and odd stages), 1 TMEM owner
// and MMA issue, 2..5 epilogue (warp w reads TMEM lanes 32 (w % 4) ..), 7..22
// transform.  The transform is latency-bound (long dependent chains per
// chunk), so it gets 16 warps: 4 per scheduler.  Every wait is
// bounded (la_sm100.cuh): one that gives up raises this file's device flag,
// read by la_device_status, and the CTA drains its copies and MMAs, frees
// its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <mutex>

#include "la_internal.cuh"
#include "la_rope.cuh"
#include "la_sm100.cuh"

namespace la {

using namespace sm100;

// Raised by a bounded wait of these kernels that gave up (0x100 | where).
__device__ unsigned int g_rope_wait_flag = 0;

namespace {

constexpr int kTabBytes = 8192;          // cos/sin table of a call
constexpr int kMinGranules = 8;          // fewest 16-token granules a reduce CTA takes

constexpr int kBox = 32 * 128;           // 32 token rows x 64 bf16 features (2 heads): 4 KiB
constexpr int kThreads = 736;
// Two warps issue the TMA loads, even and odd stages: one issuing warp moves
// at most ~27 GB/s per SM of 4-16 KiB tiles (about 4.0 TB/s over the GPU,
// measured), two reach the copy bandwidth.
constexpr int kWarpTma0 = 0, kWarpMma = 1, kWarpTma1 = 6;
constexpr int kXf0 = 224;                // first transform thread (warp 7)
constexpr int kNXf = 512;                // transform threads (warps 7..22)
constexpr int kNEpi = 128;               // epilogue threads (warps 2..5)
// Barriers that several warps release take one arrival per warp (lane 0,
// after __syncwarp orders the warp's shared-memory work before it): hundreds
// of per-thread arrivals on one barrier word serialise in shared memory.
constexpr int kXfWarps = kNXf / 32, kEpiWarps = kNEpi / 32;

// One arrival for the whole warp, after every lane's preceding work.
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// ---------------------------------------------------------------- reduce layout
// bf16 k, v: a raw stage holds k and v of 32 tokens x 4 heads (two
// 64-feature boxes each, 16 KiB); the transformed stage R phi(k) hi and lo
// (bf16, two boxes each); the MMAs read v from the raw stage.
// E4M3 codes: a raw stage holds one 128-code box of k and one of v (4 KiB
// each, 128-byte swizzle).  NVFP4: the 4 heads' E2M1 codes of k and of v (a
// 64-byte box row each: 2 KiB), then the 16-byte boxes holding their E4M3
// block scales (512 bytes each).  For both, the transformed stage holds R
// phi(k) hi and lo and the decoded v, all f16 in the bf16 path's box layout
// (24 KiB), so the raw stage is free once the transform has read it.
template <int IN>
struct RR {
    static constexpr bool Q = IN != kInBf16;               // quantised codes
    // The raw ring is as deep as shared memory allows: under load a copy takes
    // ~4 us from issue to arrival, and only the stages in flight move data.
    static constexpr int kRaw = IN == kInE4m3 ? 16 : (IN == kInNvfp4 ? 24 : 10);
    static constexpr int kRawStage = IN == kInE4m3 ? 8192 : (IN == kInNvfp4 ? 5120 : 4 * kBox);
    static constexpr int kVRaw = IN == kInE4m3 ? 4096 : (IN == kInNvfp4 ? 2048 : 2 * kBox);   // v in a raw stage
    static constexpr int kKsRaw = 4096, kVsRaw = 4608;     // NVFP4: the block-scale boxes of k, v
    static constexpr int kOp = 3;                          // transformed stages
    static constexpr int kOpStage = Q ? 6 * kBox : 4 * kBox;
    static constexpr int kOpOff = kRaw * kRawStage;
    static constexpr int kTabOff = kOpOff + kOp * kOpStage;
    static constexpr int kZOff = kTabOff + kTabBytes;      // z sums [2][4 heads][32] fp32
    static constexpr int kBarOff = kZOff + 2 * 128 * 4;
    static constexpr int kNumBars = 2 * kRaw + 2 * kOp + 2 * 4 + 1;
    static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
    static_assert(kSmem <= 232448, "reduce shared memory");
};
// Per 16 tokens two M=128 x N=128 MMAs into one accumulator: A = R phi(K)
// hi, then lo, of the 4 heads (key features as rows), B = V (value features
// as columns); the 4 diagonal 32x32 blocks of D are used.  Two accumulators
// of 128 columns.
constexpr uint32_t kRTmemCols = 256;

// ---------------------------------------------------------------- apply layout
// The apply is bound by shared-memory bandwidth, so the rotated phi(q) (hi and
// lo parts) goes to the tensor cores through tensor memory, not shared
// memory: the transform stores it with tcgen05.st and the MMA reads A from
// TMEM.  That leaves shared memory to the raw ring of q tiles (128 tokens x 2
// heads): bf16, 16 KiB each (one box of 64 features, 128-byte swizzle); E4M3
// codes, 8 KiB each (one box of 64 codes, 64-byte
// swizzle), twice as many.
constexpr int kAOp = 4;                  // transformed tiles in TMEM (hi, lo of 2 heads: 64 columns each)
constexpr int kABopBytes = 4 * 2048 + 256;              // S rows hi, lo of 2 heads, then Z_eff of 2 heads
// NVFP4 q tiles: the pair's E2M1 codes (a 32-byte box row: 4 KiB), then the
// 16-byte box holding its E4M3 block scales (2 KiB).
template <int IN>
struct AA {
    static constexpr int kTile = IN == kInE4m3 ? 128 * 64 : (IN == kInNvfp4 ? 6144 : 128 * 128);
    static constexpr int kQsOff = 4096;                          // NVFP4: the scale box in a tile
    static constexpr int kRaw = IN == kInE4m3 ? 22 : (IN == kInNvfp4 ? 29 : 11);   // raw q stages
    static constexpr int kStgOff = kRaw * kTile;                 // one [32 rows][64 bf16] staging box per epilogue warp
    static constexpr int kBopOff = kStgOff + 4 * kBox;
    static constexpr int kDenOff = kBopOff + 2 * kABopBytes;     // denominator halves [2][2 heads][2][128 rows] fp32
    static constexpr int kTabOff = kDenOff + 2 * 512 * 4;
    static constexpr int kBarOff = kTabOff + kTabBytes;
    static constexpr int kNumBars = 2 * kRaw + 2 * kAOp + 2 * 2 + 2 * 2 + 2 * 2 + 1;
    static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
    static_assert(kSmem <= 232448, "apply shared memory");
    static_assert(kABopBytes % 16 == 0 && kBopOff % 16 == 0, "bulk copies need 16-byte alignment");
};
// TMEM: two accumulators of 2 heads x 32 columns (columns 0..127), then the
// transformed tiles (columns 128..255): head hh at + 32 hh, hi at + 0, lo at
// + 16, the 16-feature K step kk at + 8 kk
constexpr uint32_t kATmemCols = 512;
constexpr uint32_t kATmemA = 128;

// ---------------------------------------------------------------- small helpers

// Two FP8 E4M3 codes (the low 16 bits of c, the low byte first) as f16x2
// (first code in the low half), exactly: every E4M3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t c) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(c & 0xFFFFu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// ReLU of one chunk of 8 E4M3 codes (features in byte order), decoded to fp32
// without the tensor's scale.  As signed bytes every negative code (sign bit
// set, -0 included) is below 0, so a signed max with 0 is ReLU on the codes.
__device__ __forceinline__ Feat8 relu_decode_e4m3(uint2 c) {
    const uint32_t w0 = __vmaxs4(c.x, 0u), w1 = __vmaxs4(c.y, 0u);
    const float2 a = f16x2_f32(e4m3x2_f16x2(w0)), b = f16x2_f32(e4m3x2_f16x2(w0 >> 16));
    const float2 cc = f16x2_f32(e4m3x2_f16x2(w1)), d = f16x2_f32(e4m3x2_f16x2(w1 >> 16));
    Feat8 f;
    f.e0 = make_float2(a.x, b.x);
    f.o0 = make_float2(a.y, b.y);
    f.e1 = make_float2(cc.x, d.x);
    f.o1 = make_float2(cc.y, d.y);
    return f;
}

// ReLU on 8 packed E2M1 codes (a nibble each): a code with its sign bit (bit
// 3) set is negative or -0 and becomes +0.
__device__ __forceinline__ uint32_t relu_e2m1x8(uint32_t w) {
    const uint32_t neg = (w >> 3) & 0x11111111u;
    return w & ~(neg * 15u);
}

// 8 E2M1 codes (element 2i in the low nibble of byte i) times their E4M3
// block scale as 8 f16 in feature order, exactly: a code value has 2
// significant bits and a scale 4, so every product (0 or 2^-10 .. 2688) is an
// f16.
__device__ __forceinline__ uint4 decode_nvfp4_8(uint32_t c, uint8_t sf) {
    const __half2 s2 = __half2half2(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sf, __NV_E4M3)));
    uint32_t o[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const __nv_fp4x2_storage_t pair = (__nv_fp4x2_storage_t)((c >> (8 * m)) & 0xFFu);
        const __half2 h = __hmul2(__half2(__nv_cvt_fp4x2_to_halfraw2(pair, __NV_E2M1)), s2);
        o[m] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// 8 f16 in feature order (4 pairs) as fp32 features.
__device__ __forceinline__ Feat8 feat_from_f16(uint4 h) {
    const float2 a = f16x2_f32(h.x), b = f16x2_f32(h.y), c = f16x2_f32(h.z), d = f16x2_f32(h.w);
    Feat8 f;
    f.e0 = make_float2(a.x, b.x);
    f.o0 = make_float2(a.y, b.y);
    f.e1 = make_float2(c.x, d.x);
    f.o1 = make_float2(c.y, d.y);
    return f;
}

// A walk over the units of a stream-K range: the unit (b, n, u) holding the
// current granule and that unit's granule range [first, end).
struct UnitWalk {
    int b, n, u;
    long long first, end;

    __device__ void start(const Sk &s, long long x) {
        sk_locate(s, x, b, n, u);
        first = sk_unit_first(s, b, n, u);
        end = first + sk_len(s, n);
    }
    // move to the unit holding x (x >= first, units in order)
    __device__ bool to(const Sk &s, long long x) {
        bool moved = false;
        while (x >= end) {
            if (++u == s.units) {
                u = 0;
                if (++n == s.nb) {
                    n = 0;
                    ++b;
                }
            }
            first = end;
            end = first + sk_len(s, n);
            moved = true;
        }
        return moved;
    }
};

// ================================================================ reduce

template <int IN>
__global__ void __launch_bounds__(kThreads, 1)
rope_reduce_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                   float *__restrict__ partials, const Plan p) {
    using C = RR<IN>;
    constexpr bool F8 = IN == kInE4m3, F4 = IN == kInNvfp4, Q = C::Q;
    constexpr int kRRaw = C::kRaw, kROp = C::kOp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *tab = smem + C::kTabOff;
    float *zbuf = reinterpret_cast<float *>(smem + C::kZOff);
    uint64_t *raw_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *raw_empty = raw_full + kRRaw;
    uint64_t *op_full = raw_empty + kRRaw;
    uint64_t *op_empty = op_full + kROp;
    uint64_t *acc_full = op_empty + kROp;   // [2]
    uint64_t *acc_empty = acc_full + 2;     // [2]
    uint64_t *z_full = acc_empty + 2;       // [2]
    uint64_t *z_empty = z_full + 2;         // [2]
    uint64_t *drain = z_empty + 2;          // only used when a wait gave up
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_word = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const Sk &S = p.skr;
    const int cta = blockIdx.x;
    const long long x_begin = sk_cta_start(S, cta), x_end = sk_cta_start(S, cta + 1);
    // k, v may come from the kernel just before this one, and the previous
    // call's combine reads the split sums this kernel writes: wait for it,
    // then let the combine be scheduled
    pdl_wait();
    pdl_trigger();
    if (x_begin >= x_end) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Llast = p.N - (p.nb - 1) * p.L;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRRaw; ++s) {
            mbar_init(&raw_full[s], 1);
            // bf16: the MMAs free a raw stage (they read v there); E4M3: the transform
            mbar_init(&raw_empty[s], Q ? kXfWarps : 1);
        }
        for (int o = 0; o < kROp; ++o) {
            mbar_init(&op_full[o], kXfWarps);
            mbar_init(&op_empty[o], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kEpiWarps);
            mbar_init(&z_full[a], kXfWarps);
            mbar_init(&z_empty[a], kEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kRTmemCols);
        tmem_relinquish();
    }
    if ((warp == kWarpTma0 || warp == kWarpTma1) && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // One segment = the part of a unit (b, block n, head group g) inside this
    // CTA's range: block tokens [tok0, tok1), its split sums in slot `slot`.
    struct Seg {
        int b, n, g, slot, tok0, tok1;
    };
    auto seg_of = [&](const UnitWalk &w, long long x) {
        Seg sg;
        sg.b = w.b;
        sg.n = w.n;
        sg.g = w.u;
        const long long e = w.end < x_end ? w.end : x_end;
        const int Ln = w.n < p.nb - 1 ? p.L : Llast;
        sg.tok0 = (int)(x - w.first) * 16;
        const int t1 = (int)(e - w.first) * 16;
        sg.tok1 = t1 < Ln ? t1 : Ln;
        sg.slot = cta - sk_cta_of(S, w.first);
        return sg;
    };
    int issued = 0;   // stages issued by this TMA warp: the last one + 1
    const int ti = warp == kWarpTma0 ? 0 : 1;

    if (warp == kWarpTma0 || warp == kWarpTma1) {
        if (lane == 0) {
            UnitWalk w;
            w.start(S, x_begin);
            bool ok = true;
            int i = 0;
            for (long long x = x_begin; ok && x < x_end; x = w.end) {
                w.to(S, x);
                const Seg sg = seg_of(w, x);
                const int nst = (sg.tok1 - sg.tok0 + 31) / 32;
                for (int st = 0; st < nst; ++st, ++i) {
                    if ((i & 1) != ti) continue;   // the other TMA warp's stage
                    const int s = i % kRRaw;
                    if (!mbar_wait(&raw_empty[s], ((uint32_t)(i / kRRaw) & 1u) ^ 1u, abort_word, &g_rope_wait_flag,
                                   1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *stg = smem + s * C::kRawStage;
                    const int row = sg.n * p.L + sg.tok0 + 32 * st;
                    const int c0 = sg.g * 128;   // features, = bytes for E4M3 codes
                    mbar_arrive_expect_tx(&raw_full[s], C::kRawStage);
                    if constexpr (F8) {
                        tma_load_3d(stg, &tm_k, &raw_full[s], c0, row, sg.b);
                        tma_load_3d(stg + C::kVRaw, &tm_v, &raw_full[s], c0, row, sg.b);
                    } else if constexpr (F4) {
                        // the group's 64 code bytes; the 16-byte box holding its 8 scale bytes
                        tma_load_3d(stg, &tm_k, &raw_full[s], sg.g * 64, row, sg.b);
                        tma_load_3d(stg + C::kVRaw, &tm_v, &raw_full[s], sg.g * 64, row, sg.b);
                        tma_load_3d(stg + C::kKsRaw, &tm_ks, &raw_full[s], (sg.g >> 1) * 16, row, sg.b);
                        tma_load_3d(stg + C::kVsRaw, &tm_vs, &raw_full[s], (sg.g >> 1) * 16, row, sg.b);
                    } else {
                        tma_load_3d(stg, &tm_k, &raw_full[s], c0, row, sg.b);
                        tma_load_3d(stg + kBox, &tm_k, &raw_full[s], c0 + 64, row, sg.b);
                        tma_load_3d(stg + C::kVRaw, &tm_v, &raw_full[s], c0, row, sg.b);
                        tma_load_3d(stg + C::kVRaw + kBox, &tm_v, &raw_full[s], c0 + 64, row, sg.b);
                    }
                    issued = i + 1;
                }
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = Q ? idesc_f16(128, 128, 1, 1) : idesc_bf16(128, 128, 1, 1);
            UnitWalk w;
            w.start(S, x_begin);
            bool ok = true;
            int i = 0, sidx = 0;
            for (long long x = x_begin; ok && x < x_end; x = w.end, ++sidx) {
                w.to(S, x);
                const Seg sg = seg_of(w, x);
                const int nst = (sg.tok1 - sg.tok0 + 31) / 32;
                const int a = sidx & 1;
                if (!mbar_wait(&acc_empty[a], ((uint32_t)(sidx >> 1) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(a * 128);
                for (int st = 0; st < nst; ++st, ++i) {
                    const int s = i % kRRaw, o = i % kROp;
                    if (!mbar_wait(&op_full[o], (uint32_t)(i / kROp) & 1u, abort_word, &g_rope_wait_flag, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t hi = smem_u32(smem + C::kOpOff + o * C::kOpStage);
                    // v: the raw stage (bf16), or the decoded box after lo (E4M3)
                    const uint32_t va = Q ? hi + 4 * kBox : smem_u32(smem + s * C::kRawStage + C::kVRaw);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        // MN-major, 128-byte swizzle: the 64-feature boxes are the MN
                        // atoms (kBox apart: v box 0, 1 for A; hi box 0, 1, lo box 0, 1
                        // for B), 8-token groups 1024 B apart, 16 tokens = 2048 B per step
                        const uint64_t dh = smem_desc(hi + kk * 2048, kBox, 1024, kLayoutSw128);
                        const uint64_t dl = smem_desc(hi + 2 * kBox + kk * 2048, kBox, 1024, kLayoutSw128);
                        const uint64_t dv = smem_desc(va + kk * 2048, kBox, 1024, kLayoutSw128);
                        mma_bf16(d, dh, dv, idesc, (st > 0 || kk > 0) ? 1u : 0u);
                        mma_bf16(d, dl, dv, idesc, 1u);
                    }
                    mma_commit(&op_empty[o]);
                    if constexpr (!Q) mma_commit(&raw_empty[s]);   // v is read from the raw stage
                }
                if (!ok) break;
                mma_commit(&acc_full[a]);
            }
            if (*abort_word) {
                // every MMA issued so far must finish before TMEM is released
                mma_commit(drain);
                final_wait(drain, 0);
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------ epilogue: warp quarter q
        // reads TMEM lanes 32q.. (the key features of head 4g + q) in columns
        // 32q.. of the accumulator (its value features); the hi and the lo MMA
        // of a stage add into the same columns
        const int q = warp & 3;
        UnitWalk w;
        w.start(S, x_begin);
        int sidx = 0;
        for (long long x = x_begin; x < x_end; x = w.end, ++sidx) {
            w.to(S, x);
            const Seg sg = seg_of(w, x);
            const int a = sidx & 1;
            const uint32_t ph = (uint32_t)(sidx >> 1) & 1u;
            bool got = mbar_wait(&acc_full[a], ph, abort_word, &g_rope_wait_flag, 4) &&
                       mbar_wait(&z_full[a], ph, abort_word, &g_rope_wait_flag, 5);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            tc_fence_after();
            float kv[32];
            tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 128 + 32 * q), kv);
            tmem_wait_ld();
            float z = zbuf[a * 128 + q * 32 + lane];
            if constexpr (Q) {
                // the sums are over the decoded values without the per-tensor
                // scales: KV = sk sv sum R phi(k^) v^, z = sk sum phi(k^)
                // (ReLU commutes with the positive scale, the rotation is linear)
                const float skv = p.sk * p.sv;
#pragma unroll
                for (int k = 0; k < 32; ++k) kv[k] *= skv;
                z *= p.sk;
            }
            tc_fence_before();
            warp_arrive(&acc_empty[a]);
            warp_arrive(&z_empty[a]);
            const int h = 4 * sg.g + q;
            float *dst = partials + ((((size_t)sg.b * p.H + h) * p.nb + sg.n) * p.skP + sg.slot) * kKVZ;
            float4 *drow = reinterpret_cast<float4 *>(dst + lane * kD);
#pragma unroll
            for (int j = 0; j < 8; ++j) drow[j] = make_float4(kv[4 * j], kv[4 * j + 1], kv[4 * j + 2], kv[4 * j + 3]);
            dst[kD * kD + lane] = z;
        }
    } else {
        // ------------------------------------------------ transform: one token row
        // (lane) per stage, feature chunk j of one head of the group.  The
        // transform warps build the cos/sin table while the first copies fly.
        const int wt = threadIdx.x - kXf0;
        build_table(tab, p, wt, kNXf);
        named_bar_sync(1, kNXf);
        const int xw = wt >> 5;
        const int j = xw & 3, head = xw >> 2;
        const int r = lane;
        // byte offset of the chunk in a stage: box head / 2, 64-byte half head % 2
        const int chunk = (head >> 1) * kBox + r * 128 + (((4 * (head & 1) + j) ^ (r & 7)) << 4);
        // E4M3: the same 8 features in the 128-code row of the raw box;
        // NVFP4: their 4 code bytes in the 64-byte row
        const int chunk8 = r * 128 + (((2 * head + (j >> 1)) ^ (r & 7)) << 4) + ((j & 1) << 3);
        const int chunk4 = r * 64 + head * 16 + j * 4;
        const GroupRec g0 = group_rec(p, 2 * j), g1 = group_rec(p, 2 * j + 1);
        Feat8 zs;
        zs.e0 = zs.o0 = zs.e1 = zs.o1 = make_float2(0.f, 0.f);
        UnitWalk w;
        w.start(S, x_begin);
        bool ok = true;
        int i = 0, sidx = 0;
        for (long long x = x_begin; x < x_end; x = w.end, ++sidx) {
            w.to(S, x);
            const Seg sg = seg_of(w, x);
            const int nst = (sg.tok1 - sg.tok0 + 31) / 32;
            Pos pq = token_pos(p, sg.n * p.L + sg.tok0 + r);   // this row's token in stage 0
            for (int st = 0; st < nst; ++st, ++i) {
                const int s = i % kRRaw, o = i % kROp;
                if (ok && !mbar_wait(&raw_full[s], (uint32_t)(i / kRRaw) & 1u, abort_word, &g_rope_wait_flag, 6))
                    ok = false;
                const int tb = sg.tok0 + 32 * st + r;   // token of this row inside the block
                const uint8_t *raw = smem + s * C::kRawStage;
                uint8_t *op = smem + C::kOpOff + o * C::kOpStage;
                uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi, vd = hi;   // rows past the segment contribute nothing
                if constexpr (F4) {
                    uint32_t ck = 0u, cv = 0u;
                    uint8_t sk = 0, sv = 0;
                    if (ok) {
                        // the scale byte of this 16-feature block in the group's half of the box row
                        const int sb = r * 16 + (sg.g & 1) * 8 + head * 2 + (j >> 1);
                        ck = *reinterpret_cast<const uint32_t *>(raw + chunk4);
                        cv = *reinterpret_cast<const uint32_t *>(raw + C::kVRaw + chunk4);
                        sk = raw[C::kKsRaw + sb];
                        sv = raw[C::kVsRaw + sb];
                    }
                    fence_proxy_async_smem();
                    warp_arrive(&raw_empty[s]);
                    if (ok && tb < sg.tok1) {
                        const Feat8 f = feat_from_f16(decode_nvfp4_8(relu_e2m1x8(ck), sk));
                        rotate_split<true>(f, tab_rec(tab, g0, pq), tab_rec(tab, g1, pq), hi, lo);
                        zs.e0 = fadd2(zs.e0, f.e0);
                        zs.o0 = fadd2(zs.o0, f.o0);
                        zs.e1 = fadd2(zs.e1, f.e1);
                        zs.o1 = fadd2(zs.o1, f.o1);
                        vd = decode_nvfp4_8(cv, sv);
                    }
                } else if constexpr (F8) {
                    uint2 ck = make_uint2(0u, 0u), cv = ck;
                    if (ok) {
                        ck = *reinterpret_cast<const uint2 *>(raw + chunk8);
                        cv = *reinterpret_cast<const uint2 *>(raw + C::kVRaw + chunk8);
                    }
                    // the raw stage may be refilled once every thread has read it
                    fence_proxy_async_smem();
                    warp_arrive(&raw_empty[s]);
                    if (ok && tb < sg.tok1) {
                        const Feat8 f = relu_decode_e4m3(ck);
                        rotate_split<true>(f, tab_rec(tab, g0, pq), tab_rec(tab, g1, pq), hi, lo);
                        zs.e0 = fadd2(zs.e0, f.e0);
                        zs.o0 = fadd2(zs.o0, f.o0);
                        zs.e1 = fadd2(zs.e1, f.e1);
                        zs.o1 = fadd2(zs.o1, f.o1);
                        vd = make_uint4(e4m3x2_f16x2(cv.x), e4m3x2_f16x2(cv.x >> 16), e4m3x2_f16x2(cv.y),
                                        e4m3x2_f16x2(cv.y >> 16));
                    }
                } else if (ok && tb < sg.tok1) {
                    const float4 t0 = tab_rec(tab, g0, pq);
                    const float4 t1 = tab_rec(tab, g1, pq);
                    Feat8 f;
                    rope_chunk(*reinterpret_cast<const uint4 *>(raw + chunk), t0, t1, hi, lo, f);
                    zs.e0 = fadd2(zs.e0, f.e0);
                    zs.o0 = fadd2(zs.o0, f.o0);
                    zs.e1 = fadd2(zs.e1, f.e1);
                    zs.o1 = fadd2(zs.o1, f.o1);
                }
                // the transformed stage is free once the MMAs of stage i - kROp are done
                if (ok && !mbar_wait(&op_empty[o], ((uint32_t)(i / kROp) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 7))
                    ok = false;
                *reinterpret_cast<uint4 *>(op + chunk) = hi;
                *reinterpret_cast<uint4 *>(op + 2 * kBox + chunk) = lo;
                if constexpr (Q) *reinterpret_cast<uint4 *>(op + 4 * kBox + chunk) = vd;
                // the generic writes of this stage before the tensor cores read it
                fence_proxy_async_smem();
                warp_arrive(&op_full[o]);
                pos_step(p, pq, 32);
            }
            // the segment's z: this thread's 8 features summed over the 32 rows
            float zv[8] = {zs.e0.x, zs.o0.x, zs.e0.y, zs.o0.y, zs.e1.x, zs.o1.x, zs.e1.y, zs.o1.y};
            zs.e0 = zs.o0 = zs.e1 = zs.o1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) zv[k] += __shfl_xor_sync(0xffffffffu, zv[k], off);
            const int a = sidx & 1;
            if (ok && !mbar_wait(&z_empty[a], ((uint32_t)(sidx >> 1) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 8))
                ok = false;
            if (lane == 0) {
                float4 *zz = reinterpret_cast<float4 *>(zbuf + a * 128 + head * 32 + 8 * j);
                zz[0] = make_float4(zv[0], zv[1], zv[2], zv[3]);
                zz[1] = make_float4(zv[4], zv[5], zv[6], zv[7]);
            }
            warp_arrive(&z_full[a]);
        }
    }

    // teardown: nothing may still write this CTA's shared memory or TMEM
    if ((warp == kWarpTma0 || warp == kWarpTma1) && lane == 0 && *abort_word) {
        for (int i = issued - kRRaw < 0 ? 0 : issued - kRRaw; i < issued; ++i)
            if ((i & 1) == ti) final_wait(&raw_full[i % kRRaw], (uint32_t)(i / kRRaw) & 1u);
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kRTmemCols);
    }
}

// ================================================================ apply

template <int IN>
__global__ void __launch_bounds__(kThreads, 1)
rope_apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qs,
                  const __grid_constant__ CUtensorMap tm_out, __nv_bfloat16 *__restrict__ out,
                  const uint8_t *__restrict__ bop, const float *__restrict__ seff, const Plan p) {
    using C = AA<IN>;
    constexpr bool F8 = IN == kInE4m3, F4 = IN == kInNvfp4, Q = IN != kInBf16;
    constexpr int kARaw = C::kRaw, kATile = C::kTile;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *tab = smem + C::kTabOff;
    uint8_t *bops = smem + C::kBopOff;
    float *den_s = reinterpret_cast<float *>(smem + C::kDenOff);
    uint64_t *raw_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *raw_empty = raw_full + kARaw;
    uint64_t *op_full = raw_empty + kARaw;
    uint64_t *op_empty = op_full + kAOp;
    uint64_t *acc_full = op_empty + kAOp;   // [2]
    uint64_t *acc_empty = acc_full + 2;     // [2]
    uint64_t *den_full = acc_empty + 2;     // [2]
    uint64_t *den_empty = den_full + 2;     // [2]
    uint64_t *bop_full = den_empty + 2;     // [2]
    uint64_t *bop_empty = bop_full + 2;     // [2]
    uint64_t *drain = bop_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_word = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const Sk &S = p.ska;
    const int cta = blockIdx.x;
    const long long x_begin = sk_cta_start(S, cta), x_end = sk_cta_start(S, cta + 1);
    // the next kernel may be scheduled now: it waits for this grid before it
    // touches anything this grid reads or writes
    pdl_trigger();
    if (x_begin >= x_end) return;
    const int ntiles = (int)(x_end - x_begin);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Llast = p.N - (p.nb - 1) * p.L;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kARaw; ++s) {
            mbar_init(&raw_full[s], 1);
            mbar_init(&raw_empty[s], kXfWarps);
        }
        for (int o = 0; o < kAOp; ++o) {
            mbar_init(&op_full[o], kXfWarps);
            mbar_init(&op_empty[o], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kEpiWarps);
            mbar_init(&den_full[a], kXfWarps);
            mbar_init(&den_empty[a], kEpiWarps);
            mbar_init(&bop_full[a], 1);
            mbar_init(&bop_empty[a], 1);
        }
        mbar_init(drain, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kATmemCols);
        tmem_relinquish();
    }
    if ((warp == kWarpTma0 || warp == kWarpTma1) && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_out);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0, bops_issued = 0;   // by this TMA warp: the last q tile + 1, operands loaded
    const int ti = warp == kWarpTma0 ? 0 : 1;

    if (warp == kWarpTma0 || warp == kWarpTma1) {
        if (lane == 0) {
            auto load_q = [&](const UnitWalk &w, long long x, int i) {
                const int s = i % kARaw;
                const int row = w.n * p.L + (int)(x - w.first) * 128;
                mbar_arrive_expect_tx(&raw_full[s], kATile);
                if constexpr (F4) {
                    // the pair's 32 code bytes; the 16-byte box holding its 4 scale bytes
                    tma_load_3d(smem + s * kATile, &tm_q, &raw_full[s], w.u * 32, row, w.b);
                    tma_load_3d(smem + s * kATile + C::kQsOff, &tm_qs, &raw_full[s], (w.u >> 2) * 16, row, w.b);
                } else {
                    tma_load_3d(smem + s * kATile, &tm_q, &raw_full[s], w.u * 64, row, w.b);
                }
                issued = i + 1;
            };
            // the packed operand rows of S_eff (hi, lo) and Z_eff of the unit's 2 heads
            auto load_bop = [&](const UnitWalk &w, int kb) -> bool {
                const int bi = kb & 1;
                if (!mbar_wait(&bop_empty[bi], ((uint32_t)(kb >> 1) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 11))
                    return false;
                uint8_t *dst = bops + bi * kABopBytes;
                mbar_arrive_expect_tx(&bop_full[bi], kABopBytes);
                for (int hh = 0; hh < 2; ++hh) {
                    const size_t bhn = ((size_t)w.b * p.H + 2 * w.u + hh) * p.nb + w.n;
                    const uint8_t *src = bop + bhn * 2 * kOpBytes;
                    bulk_load(dst + hh * 4096, src, 2048, &bop_full[bi]);
                    bulk_load(dst + hh * 4096 + 2048, src + kOpBytes, 2048, &bop_full[bi]);
                    bulk_load(dst + 8192 + hh * 128, seff + bhn * kKVZ + kD * kD, 128, &bop_full[bi]);
                }
                bops_issued = kb + 1;
                return true;
            };
            // q is an input of the call, complete before this call's reduce
            // started: the first tiles are fetched while the combine still runs.
            // This warp takes the q tiles i with i % 2 == ti; warp 0 also loads
            // each unit's state operand once the combine is done.
            const int pre = ntiles < kARaw ? ntiles : kARaw;
            UnitWalk w;
            w.start(S, x_begin);
            for (int i = 0; i < pre; ++i) {
                w.to(S, x_begin + i);
                if ((i & 1) == ti) load_q(w, x_begin + i, i);
            }
            if (ti == 0) pdl_wait();   // the packed operand and Z_eff are written by the combine
            w.start(S, x_begin);
            int kb = 0;
            for (int i = 0; i < ntiles; ++i) {
                const long long x = x_begin + i;
                if (w.to(S, x) || i == 0) {
                    if (ti == 0 && !load_bop(w, kb++)) break;
                }
                if (i < pre || (i & 1) != ti) continue;
                const int s = i % kARaw;
                if (!mbar_wait(&raw_empty[s], ((uint32_t)(i / kARaw) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 12))
                    break;
                load_q(w, x, i);
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, 32, 0, 0);
            UnitWalk w;
            w.start(S, x_begin);
            int kb = -1;
            for (int i = 0; i < ntiles; ++i) {
                const long long x = x_begin + i;
                if (w.to(S, x) || i == 0) {
                    ++kb;
                    if (!mbar_wait(&bop_full[kb & 1], (uint32_t)(kb >> 1) & 1u, abort_word, &g_rope_wait_flag, 13))
                        break;
                }
                const int a = i & 1, o = i % kAOp;
                if (!mbar_wait(&acc_empty[a], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 14)) break;
                if (!mbar_wait(&op_full[o], (uint32_t)(i / kAOp) & 1u, abort_word, &g_rope_wait_flag, 15)) break;
                tc_fence_after();
                const uint32_t qa = tmem + kATmemA + (uint32_t)(o * 64);
                const uint32_t ba = smem_u32(bops + (kb & 1) * kABopBytes);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t d = tmem + (uint32_t)(a * 64 + hh * 32);
                    // (A part, B part): hi.hi, hi.lo, lo.hi
#pragma unroll
                    for (int prod = 0; prod < 3; ++prod) {
                        const int apart = prod == 2 ? 1 : 0, bpart = prod == 1 ? 1 : 0;
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            // A in TMEM: token row = lane, 8 columns per 16 features
                            const uint32_t ta = qa + (uint32_t)(hh * 32 + apart * 16 + kk * 8);
                            // B: K-major, no swizzle, core matrices 128 B apart along K,
                            // 8-row groups 512 B apart; 16 features = 256 bytes per step
                            const uint64_t db =
                                smem_desc(ba + hh * 4096 + bpart * 2048 + kk * 256, 128, 512, kLayoutNone);
                            mma_bf16_ta(d, ta, db, idesc, (prod | kk) ? 1u : 0u);
                        }
                    }
                }
                mma_commit(&op_empty[o]);
                mma_commit(&acc_full[a]);
                if (x + 1 == w.end || i + 1 == ntiles) mma_commit(&bop_empty[kb & 1]);
            }
            if (*abort_word) {
                mma_commit(drain);
                final_wait(drain, 0);
            }
        }
    } else if (warp >= 7) {
        // ------------------------------------------------ transform: token row r of
        // the tile, feature chunks 2 jh and 2 jh + 1 of head hh.  A warp writes
        // TMEM lanes 32 (warp % 4) .., so its rows are that quarter of the tile.
        // The transform warps build the cos/sin table while the first q tiles fly.
        const int wt = threadIdx.x - kXf0;
        build_table(tab, p, wt, kNXf);
        named_bar_sync(1, kNXf);
        const int xw = (warp - 7) >> 2;   // 0..3: which of the 4 warps of a lane quarter
        const int hh = xw >> 1, jh = xw & 1;
        const int r = 32 * (warp & 3) + lane;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const GroupRec gr[2][2] = {{group_rec(p, 4 * jh), group_rec(p, 4 * jh + 1)},
                                   {group_rec(p, 4 * jh + 2), group_rec(p, 4 * jh + 3)}};
        float2 ze[2][2], zo[2][2];   // Z_eff of head hh: chunk, pairs (a, b) / (c, d), even / odd features
        UnitWalk w;
        w.start(S, x_begin);
        bool ok = true;
        int kb = -1;
        Pos pq{};
        for (int i = 0; i < ntiles; ++i) {
            const long long x = x_begin + i;
            w.to(S, x);
            const int row0 = (int)(x - w.first) * 128;
            if (i == 0 || x == w.first) {   // the first tile of a unit in this CTA
                ++kb;
                if (ok && !mbar_wait(&bop_full[kb & 1], (uint32_t)(kb >> 1) & 1u, abort_word, &g_rope_wait_flag, 16))
                    ok = false;
                const float4 *zsrc = reinterpret_cast<const float4 *>(bops + (kb & 1) * kABopBytes + 8192 + hh * 128);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int j = 2 * jh + c;
                    const float4 u0 = zsrc[2 * j], u1 = zsrc[2 * j + 1];   // features 8j .. 8j + 7
                    ze[c][0] = make_float2(u0.x, u0.z);
                    zo[c][0] = make_float2(u0.y, u0.w);
                    ze[c][1] = make_float2(u1.x, u1.z);
                    zo[c][1] = make_float2(u1.y, u1.w);
                }
                pq = token_pos(p, w.n * p.L + row0 + r);
            } else {
                pos_step(p, pq, 128);
            }
            const int s = i % kARaw, o = i % kAOp, a = i & 1;
            const int Ln = w.n < p.nb - 1 ? p.L : Llast;
            const bool valid = r < Ln - row0;
            if (ok && !mbar_wait(&raw_full[s], (uint32_t)(i / kARaw) & 1u, abort_word, &g_rope_wait_flag, 17)) ok = false;
            uint4 xq[2];
            if constexpr (F4) {
                // the 16 codes of block jh of head hh (8 bytes of the 32-byte row) and
                // their scale byte; ReLU on the codes, then f16 values
                const uint8_t *raw = smem + s * kATile;
                uint2 c = make_uint2(0u, 0u);
                uint8_t sf = 0;
                if (ok && valid) {
                    c = *reinterpret_cast<const uint2 *>(raw + r * 32 + hh * 16 + jh * 8);
                    sf = raw[C::kQsOff + r * 16 + (w.u & 3) * 4 + hh * 2 + jh];
                }
                xq[0] = decode_nvfp4_8(relu_e2m1x8(c.x), sf);
                xq[1] = decode_nvfp4_8(relu_e2m1x8(c.y), sf);
            } else if constexpr (F8) {
                // 16 codes (features 16 jh ..) of the 64-code row, 64-byte swizzle:
                // 16-byte chunk c of row r at c ^ ((r / 2) % 4)
                const uint8_t *raw = smem + s * kATile + r * 64;
                const uint4 x8 = (ok && valid)
                                     ? *reinterpret_cast<const uint4 *>(raw + (((2 * hh + jh) ^ ((r >> 1) & 3)) << 4))
                                     : make_uint4(0u, 0u, 0u, 0u);
                xq[0] = make_uint4(x8.x, x8.y, 0u, 0u);
                xq[1] = make_uint4(x8.z, x8.w, 0u, 0u);
            } else {
                const uint8_t *raw = smem + s * kATile + r * 128;
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    xq[c] = (ok && valid)
                                ? *reinterpret_cast<const uint4 *>(raw + (((4 * hh + 2 * jh + c) ^ (r & 7)) << 4))
                                : make_uint4(0u, 0u, 0u, 0u);
            }
            // the raw stage may be refilled as soon as every thread has read it:
            // order these generic reads before the async proxy's refill
            fence_proxy_async_smem();
            warp_arrive(&raw_empty[s]);
            uint4 hi[2], lo[2];
            float2 den = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                hi[c] = lo[c] = make_uint4(0u, 0u, 0u, 0u);
                if (ok && valid) {
                    Feat8 f;
                    if constexpr (F4) {
                        f = feat_from_f16(xq[c]);   // without the tensor's scale (the epilogue applies it)
                        rotate_split<false>(f, tab_rec(tab, gr[c][0], pq), tab_rec(tab, gr[c][1], pq), hi[c], lo[c]);
                    } else if constexpr (F8) {
                        // the codes without the tensor's scale (the epilogue applies it)
                        f = relu_decode_e4m3(make_uint2(xq[c].x, xq[c].y));
                        rotate_split<false>(f, tab_rec(tab, gr[c][0], pq), tab_rec(tab, gr[c][1], pq), hi[c], lo[c]);
                    } else {
                        rope_chunk(xq[c], tab_rec(tab, gr[c][0], pq), tab_rec(tab, gr[c][1], pq), hi[c], lo[c], f);
                    }
                    // the denominator takes the unrotated phi(q)
                    den = ffma2(f.e0, ze[c][0], den);
                    den = ffma2(f.o0, zo[c][0], den);
                    den = ffma2(f.e1, ze[c][1], den);
                    den = ffma2(f.o1, zo[c][1], den);
                }
            }
            // the transformed tile is free once the MMAs of tile i - kAOp are done
            if (ok && !mbar_wait(&op_empty[o], ((uint32_t)(i / kAOp) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 18))
                ok = false;
            if (ok && !mbar_wait(&den_empty[a], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 19))
                ok = false;
            // the warp's lanes store together: a wait that gave up in one lane stops the warp
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                // features 16 jh .. 16 jh + 15 of head hh: TMEM columns 8 jh .. 8 jh + 7 of
                // the head's hi and lo parts (two features per column)
                const uint32_t ta = tmem + lane_off + kATmemA + (uint32_t)(o * 64 + hh * 32 + 8 * jh);
                const uint32_t vh[8] = {hi[0].x, hi[0].y, hi[0].z, hi[0].w, hi[1].x, hi[1].y, hi[1].z, hi[1].w};
                const uint32_t vl[8] = {lo[0].x, lo[0].y, lo[0].z, lo[0].w, lo[1].x, lo[1].y, lo[1].z, lo[1].w};
                tmem_st8(ta, vh);
                tmem_st8(ta + 16, vl);
                tmem_wait_st();
            }
            den_s[a * 512 + (2 * hh + jh) * 128 + r] = den.x + den.y;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&op_full[o]);
                mbar_arrive(&den_full[a]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5, one
        // head at a time
        const int q = warp & 3;
        const int r = 32 * q + lane;               // token row of this thread in a tile
        uint8_t *sb = smem + C::kStgOff + q * kBox;  // this warp's staging box
        UnitWalk w;
        w.start(S, x_begin);
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const long long x = x_begin + i;
            w.to(S, x);
            const int a = i & 1;
            const uint32_t aph = (uint32_t)(i >> 1) & 1u;
            bool got = ok && mbar_wait(&acc_full[a], aph, abort_word, &g_rope_wait_flag, 20) &&
                       mbar_wait(&den_full[a], aph, abort_word, &g_rope_wait_flag, 21);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
            const int Ln = w.n < p.nb - 1 ? p.L : Llast;
            const int row0 = (int)(x - w.first) * 128;
            const int blk0 = w.n * p.L;                // first token of the block in the call
            // TMA store of the warp's 32 rows unless they run into the next block
            // (rows past the end of the tensor are clipped by TMA)
            const bool boxed = row0 + 32 * q + 32 <= Ln || blk0 + Ln == p.N;
            if (got) {
                tc_fence_after();
                if (boxed) {
                    if (lane == 0) bulk_wait_read<0>();   // the last store from this box has read it
                    __syncwarp();
                }
                const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 64);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tmem_ld32(base + hh * 32, v);
                    tmem_wait_ld();
                    // the sum of the two halves of the denominator, in a fixed order
                    const float den = den_s[a * 512 + (2 * hh) * 128 + r] + den_s[a * 512 + (2 * hh + 1) * 128 + r];
                    // E4M3, NVFP4: out = sq num^ / (sq den^ + eps), num^ and den^ without sq
                    const float iv = Q ? p.sq / (p.sq * den + p.eps) : 1.0f / (den + p.eps);
                    const float2 inv = make_float2(iv, iv);
                    uint4 y[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 y0 = fmul2(make_float2(v[8 * c], v[8 * c + 1]), inv);
                        const float2 y1 = fmul2(make_float2(v[8 * c + 2], v[8 * c + 3]), inv);
                        const float2 y2 = fmul2(make_float2(v[8 * c + 4], v[8 * c + 5]), inv);
                        const float2 y3 = fmul2(make_float2(v[8 * c + 6], v[8 * c + 7]), inv);
                        y[c] = make_uint4(pack_bf2(y0.x, y0.y), pack_bf2(y1.x, y1.y), pack_bf2(y2.x, y2.y),
                                          pack_bf2(y3.x, y3.y));
                    }
                    if (boxed) {
#pragma unroll
                        for (int c = 0; c < 4; ++c)   // logical chunk 4 hh + c, 128-byte swizzle (row % 8 == lane % 8)
                            *reinterpret_cast<uint4 *>(sb + lane * 128 + (((4 * hh + c) ^ (lane & 7)) << 4)) = y[c];
                    } else if (row0 + r < Ln) {
                        // a short last tile of a block that is not the last of the
                        // tensor: the rows after the block belong to the next block
                        uint4 *dst = reinterpret_cast<uint4 *>(
                            out + (((size_t)w.b * p.N + blk0 + row0 + r) * p.H + 2 * w.u + hh) * kD);
#pragma unroll
                        for (int c = 0; c < 4; ++c) dst[c] = y[c];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&acc_empty[a]);
                mbar_arrive(&den_empty[a]);
            }
            if (got && boxed) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&tm_out, sb, w.u * 64, blk0 + row0 + 32 * q, w.b);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    if ((warp == kWarpTma0 || warp == kWarpTma1) && lane == 0 && *abort_word) {
        for (int kb = bops_issued - 2 < 0 ? 0 : bops_issued - 2; kb < bops_issued; ++kb)
            final_wait(&bop_full[kb & 1], (uint32_t)(kb >> 1) & 1u);
        for (int i = issued - kARaw < 0 ? 0 : issued - kARaw; i < issued; ++i)
            if ((i & 1) == ti) final_wait(&raw_full[i % kARaw], (uint32_t)(i / kARaw) & 1u);
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kATmemCols);
    }
}

bool smem_ready() {
    static std::once_flag once;
    static bool ok = false;
    std::call_once(once, [] {
        ok = set_smem((const void *)rope_reduce_kernel<kInBf16>, RR<kInBf16>::kSmem) &&
             set_smem((const void *)rope_apply_kernel<kInBf16>, AA<kInBf16>::kSmem) &&
             set_smem((const void *)rope_reduce_kernel<kInE4m3>, RR<kInE4m3>::kSmem) &&
             set_smem((const void *)rope_apply_kernel<kInE4m3>, AA<kInE4m3>::kSmem) &&
             set_smem((const void *)rope_reduce_kernel<kInNvfp4>, RR<kInNvfp4>::kSmem) &&
             set_smem((const void *)rope_apply_kernel<kInNvfp4>, AA<kInNvfp4>::kSmem);
    });
    return ok;
}

}  // namespace

// ================================================================ host side

void plan_rope_sk(Plan &p) {
    p.skP = 0;
    p.skr = Sk{};
    p.ska = Sk{};
    if (p.H <= 0 || p.H % 4 != 0 || p.nb < 1 || p.L < 1 || p.B < 1) return;
    const int Llast = p.N - (p.nb - 1) * p.L;
    Sk r{};
    r.units = p.H / 4;
    r.nb = p.nb;
    r.g_full = (p.L + 15) / 16;
    r.g_last = (Llast + 15) / 16;
    r.C = 1;
    r.total = (long long)p.B * sk_per_b(r);
    // at least kMinGranules per CTA: below that a CTA's fixed costs (table,
    // barriers, TMEM) and its split sums outweigh its share of the tokens
    const long long want = r.total / kMinGranules > 0 ? r.total / kMinGranules : 1;
    r.C = (int)(want < kSmCount ? want : kSmCount);
    // a unit of g granules meets at most 1 + ceil((g - 1) / q) CTA ranges when
    // every range holds at least q granules
    const long long qg = r.total / r.C;
    p.skP = 1 + (int)((r.g_full - 1 + qg - 1) / qg);
    Sk a{};
    a.units = p.H / 2;
    a.nb = p.nb;
    a.g_full = (p.L + 127) / 128;
    a.g_last = (Llast + 127) / 128;
    a.C = 1;
    a.total = (long long)p.B * sk_per_b(a);
    a.C = (int)(a.total < kSmCount ? a.total : kSmCount);
    p.skr = r;
    p.ska = a;
}

void plan_rope_table(Plan &p) {
    p.tab_bytes = 0;
    if (!p.rope || p.Hg <= 0 || p.Wg <= 0) return;
    // each group of 4 features (2 pairs) must lie on one axis
    int per_axis[3] = {0, 0, 0}, index[8];
    for (int m = 0; m < 8; ++m) {
        const int ax = p.axis[2 * m];
        if (p.axis[2 * m + 1] != ax || ax < 0 || ax > 2) return;
        p.hc_axis[m] = ax;
        index[m] = per_axis[ax]++;
    }
    const long long hw = (long long)p.Hg * p.Wg;
    const long long frames = (p.N - 1) / hw + 1;
    if (frames > 1 << 20) return;
    p.tab_frames = (int)frames;
    const long long len[3] = {frames, p.Hg, p.Wg};
    long long off[4] = {0, 0, 0, 0};
    for (int ax = 0; ax < 3; ++ax) off[ax + 1] = off[ax] + len[ax] * 16 * per_axis[ax];
    if (off[3] > kTabBytes) return;
    for (int m = 0; m < 8; ++m) {
        const int ax = p.hc_axis[m];
        p.hc_stride[m] = 16 * per_axis[ax];
        p.hc_base[m] = (int)off[ax] + 16 * index[m];
    }
    p.tab_bytes = (int)off[3];
}

bool tc_rope_fits(const Plan &p) { return p.rope && p.tab_bytes > 0 && p.H % 4 == 0 && p.skr.C > 0; }

int launch_reduce_rope_tc(const void *k, const void *v, float *partials, const Plan &p, cudaStream_t s) {
    if (!smem_ready() || !tc_rope_fits(p) || !p.sk_layout) return -1;
    CUtensorMap mk, mv, mks, mvs;
    const unsigned grid = (unsigned)p.skr.C;
    const long long row = (long long)p.H * kD;   // features (bf16), codes (E4M3)
    if (p.f4) {
        // NVFP4: 64-byte boxes of the group's codes, 16-byte boxes of scales
        if (p.H % 8 != 0 || !make_u8_map(&mk, k, p.B, p.N, row / 2, 64, 32, 0) ||
            !make_u8_map(&mv, v, p.B, p.N, row / 2, 64, 32, 0) ||
            !make_u8_map(&mks, p.sfk, p.B, p.N, row / 16, 16, 32, 0) ||
            !make_u8_map(&mvs, p.sfv, p.B, p.N, row / 16, 16, 32, 0))
            return -1;
        return launch_pdl(rope_reduce_kernel<kInNvfp4>, grid, kThreads, RR<kInNvfp4>::kSmem, s, mk, mv, mks, mvs,
                          partials, p)
                   ? 1
                   : -1;
    }
    if (p.f8) {
        // E4M3 codes: boxes of the 4 heads' 128 codes x 32 tokens, 128-byte swizzle
        if (!make_u8_map(&mk, k, p.B, p.N, row, 128, 32, 128) || !make_u8_map(&mv, v, p.B, p.N, row, 128, 32, 128))
            return -1;
        return launch_pdl(rope_reduce_kernel<kInE4m3>, grid, kThreads, RR<kInE4m3>::kSmem, s, mk, mv, mk, mv,
                          partials, p)
                   ? 1
                   : -1;
    }
    if (!make_bf16_map(&mk, k, p.B, p.N, p.H, 32) || !make_bf16_map(&mv, v, p.B, p.N, p.H, 32)) return -1;
    return launch_pdl(rope_reduce_kernel<kInBf16>, grid, kThreads, RR<kInBf16>::kSmem, s, mk, mv, mk, mv, partials,
                      p)
               ? 1
               : -1;
}

int launch_apply_rope_tc(const void *q, void *out, const void *bop, const float *seff, const Plan &p,
                         cudaStream_t s) {
    if (!smem_ready() || !tc_rope_fits(p)) return -1;
    CUtensorMap mq, mqs, mo;
    const unsigned grid = (unsigned)p.ska.C;
    const long long row = (long long)p.H * kD;
    if (!make_bf16_map(&mo, out, p.B, p.N, p.H, 32)) return -1;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
    const uint8_t *b = static_cast<const uint8_t *>(bop);
    if (p.f4) {
        // NVFP4: 32-byte boxes of a head pair's codes x 128 tokens, 16-byte boxes of scales
        if (p.H % 8 != 0 || !make_u8_map(&mq, q, p.B, p.N, row / 2, 32, 128, 0) ||
            !make_u8_map(&mqs, p.sfq, p.B, p.N, row / 16, 16, 128, 0))
            return -1;
        return launch_pdl(rope_apply_kernel<kInNvfp4>, grid, kThreads, AA<kInNvfp4>::kSmem, s, mq, mqs, mo, o, b,
                          seff, p)
                   ? 1
                   : -1;
    }
    if (p.f8) {
        // E4M3 codes: boxes of a head pair's 64 codes x 128 tokens, 64-byte swizzle
        if (!make_u8_map(&mq, q, p.B, p.N, row, 64, 128, 64)) return -1;
        return launch_pdl(rope_apply_kernel<kInE4m3>, grid, kThreads, AA<kInE4m3>::kSmem, s, mq, mq, mo, o, b, seff,
                          p)
                   ? 1
                   : -1;
    }
    if (!make_bf16_map(&mq, q, p.B, p.N, p.H, 128)) return -1;
    return launch_pdl(rope_apply_kernel<kInBf16>, grid, kThreads, AA<kInBf16>::kSmem, s, mq, mq, mo, o, b, seff, p)
               ? 1
               : -1;
}

int read_and_clear_rope_flag(unsigned *flag_out) {
    unsigned zero = 0;
    if (cudaMemcpyFromSymbol(flag_out, g_rope_wait_flag, sizeof(unsigned)) != cudaSuccess) return -1;
    if (*flag_out && cudaMemcpyToSymbol(g_rope_wait_flag, &zero, sizeof(unsigned)) != cudaSuccess) return -1;
    return 0;
}

}  // namespace la
