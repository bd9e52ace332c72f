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
// stages (160 KiB in the reduce, 112 KiB in the apply) separate from the
// transformed operands the tensor cores read, so that a raw q stage is free
// as soon as the transform has read it.  The cos/sin table holds records of
// two feature pairs (cos a, cos b, sin a, sin b) per position of each axis;
// a transform thread owns one token row, so the 8 lanes of a shared-memory
// phase read 8 consecutive rows: distinct 16-byte chunks of the swizzled
// tiles, and for the column axis distinct consecutive records.
//
// Warp roles (448 threads): 0 TMA, 1 TMEM owner and MMA issue, 2..5 epilogue
// (warp w reads TMEM lanes 32 (w % 4) ..), 6..13 transform.  Every wait is
// bounded (la_sm100.cuh): one that gives up raises this file's device flag,
// read by la_device_status, and the CTA drains its copies and MMAs, frees
// its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "la_internal.cuh"
#include "la_sm100.cuh"

namespace la {

using namespace sm100;

// Raised by a bounded wait of these kernels that gave up (0x100 | where).
__device__ unsigned int g_rope_wait_flag = 0;

namespace {

constexpr int kTabBytes = 8192;          // cos/sin table of a call
constexpr int kMinGranules = 8;          // fewest 16-token granules a reduce CTA takes
constexpr int kBox = 32 * 128;           // 32 token rows x 64 bf16 features (2 heads): 4 KiB
constexpr int kThreads = 448;
constexpr int kWarpTma = 0, kWarpMma = 1;
constexpr int kXf0 = 192;                // first transform thread (warp 6)
constexpr int kNXf = 256;                // transform threads
constexpr int kNEpi = 128;               // epilogue threads (warps 2..5)

// ---------------------------------------------------------------- reduce layout
constexpr int kRRaw = 10;                // raw stages: k (2 boxes) and v (2 boxes) of 32 tokens x 4 heads
constexpr int kROp = 3;                  // transformed stages: R phi(k) hi (2 boxes), lo (2 boxes)
constexpr int kRStage = 4 * kBox;        // 16 KiB, raw and transformed alike
constexpr int kROpOff = kRRaw * kRStage;
constexpr int kRTabOff = kROpOff + kROp * kRStage;
constexpr int kRZOff = kRTabOff + kTabBytes;             // z sums [2][4 heads][32] fp32
constexpr int kRBarOff = kRZOff + 2 * 128 * 4;
constexpr int kRNumBars = 2 * kRRaw + 2 * kROp + 2 * 4 + 1;
constexpr int kRSmem = kRBarOff + kRNumBars * 8 + 16 + 1024;
constexpr uint32_t kRTmemCols = 256;     // two accumulators of 128 columns
static_assert(kRSmem <= 232448, "reduce shared memory");

// ---------------------------------------------------------------- apply layout
constexpr int kATile = 128 * 128;        // 128 tokens x 64 bf16 features (2 heads): 16 KiB
constexpr int kARaw = 7;                 // raw q stages
constexpr int kAOp = 2;                  // transformed tiles: R phi(q) hi, then lo
constexpr int kAOpOff = kARaw * kATile;
constexpr int kAStgOff = kAOpOff + kAOp * 2 * kATile;   // one [32 rows][64 bf16] staging box per epilogue warp
constexpr int kABopBytes = 4 * 2048 + 256;              // S rows hi, lo of 2 heads, then Z_eff of 2 heads
constexpr int kABopOff = kAStgOff + 4 * kBox;
constexpr int kADenOff = kABopOff + 2 * kABopBytes;     // denominators [2][2 heads][128 rows] fp32
constexpr int kATabOff = kADenOff + 2 * 256 * 4;
constexpr int kABarOff = kATabOff + kTabBytes;
constexpr int kANumBars = 2 * kARaw + 2 * kAOp + 2 * 2 + 2 * 2 + 2 * 2 + 1;
constexpr int kASmem = kABarOff + kANumBars * 8 + 16 + 1024;
constexpr uint32_t kATmemCols = 128;     // two accumulators of 2 heads x 32 columns
static_assert(kASmem <= 232448, "apply shared memory");
static_assert(kABopBytes % 16 == 0 && kABopOff % 16 == 0, "bulk copies need 16-byte alignment");

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// The ReLU'd features of one 16-byte chunk (4 feature pairs a, b, c, d) as
// fp32: e = even features (x_2i), o = odd features (x_2i+1), two pairs each.
struct Feat8 {
    float2 e0, o0;   // pairs a, b
    float2 e1, o1;   // pairs c, d
};

// ReLU one chunk of 8 bf16 (4 feature pairs), rotate pair (x0, x1) by its
// (cos, sin) to (x0 cos - x1 sin, x0 sin + x1 cos), and split the rotated
// values into bf16 hi = RN(y) and lo = RN(y - hi).  t0 = (cos a, cos b,
// sin a, sin b), t1 the same for pairs c, d.  f receives phi(x).
__device__ __forceinline__ void rope_chunk(uint4 x, float4 t0, float4 t1, uint4 &hi, uint4 &lo, Feat8 &f) {
    const uint32_t wa = relu2(x.x), wb = relu2(x.y), wc = relu2(x.z), wd = relu2(x.w);
    f.e0 = make_float2(bf_lo(wa), bf_lo(wb));
    f.o0 = make_float2(bf_hi(wa), bf_hi(wb));
    f.e1 = make_float2(bf_lo(wc), bf_lo(wd));
    f.o1 = make_float2(bf_hi(wc), bf_hi(wd));
    const float2 c0 = make_float2(t0.x, t0.y), s0 = make_float2(t0.z, t0.w);
    const float2 c1 = make_float2(t1.x, t1.y), s1 = make_float2(t1.z, t1.w);
    const float2 ye0 = ffma2(f.o0, make_float2(-s0.x, -s0.y), fmul2(f.e0, c0));
    const float2 yo0 = ffma2(f.o0, c0, fmul2(f.e0, s0));
    const float2 ye1 = ffma2(f.o1, make_float2(-s1.x, -s1.y), fmul2(f.e1, c1));
    const float2 yo1 = ffma2(f.o1, c1, fmul2(f.e1, s1));
    hi = make_uint4(pack_bf2(ye0.x, yo0.x), pack_bf2(ye0.y, yo0.y), pack_bf2(ye1.x, yo1.x), pack_bf2(ye1.y, yo1.y));
    // y - hi is exact in fp32
    const float2 re0 = fsub2(ye0, make_float2(bf_lo(hi.x), bf_lo(hi.y)));
    const float2 ro0 = fsub2(yo0, make_float2(bf_hi(hi.x), bf_hi(hi.y)));
    const float2 re1 = fsub2(ye1, make_float2(bf_lo(hi.z), bf_lo(hi.w)));
    const float2 ro1 = fsub2(yo1, make_float2(bf_hi(hi.z), bf_hi(hi.w)));
    lo = make_uint4(pack_bf2(re0.x, ro0.x), pack_bf2(re0.y, ro0.y), pack_bf2(re1.x, ro1.x), pack_bf2(re1.y, ro1.y));
}

// The (cos, sin) records of every position of the call: for each of the 8
// groups of 4 features m, its two pairs 2m, 2m+1 at every position along the
// group's axis (frames of the call, rows, columns), at the byte offsets the
// host planned.
__device__ void build_table(uint8_t *tab, const Plan &p, int tid, int nthr) {
#pragma unroll 1
    for (int m = 0; m < 8; ++m) {
        const int ax = p.hc_axis[m];
        const int len = ax == 0 ? p.tab_frames : (ax == 1 ? p.Hg : p.Wg);
        for (int pos = tid; pos < len; pos += nthr) {
            const int apos = ax == 0 ? p.t_offset + pos : pos;
            float sa, ca, sb, cb;
            sincosf((float)apos * p.theta[2 * m], &sa, &ca);
            sincosf((float)apos * p.theta[2 * m + 1], &sb, &cb);
            *reinterpret_cast<float4 *>(tab + p.hc_base[m] + pos * p.hc_stride[m]) = make_float4(ca, cb, sa, sb);
        }
    }
}

// Position of token jg of the call along the axes (frame relative to token 0
// of the call, row, column).
struct Pos {
    int f, h, w;
};

__device__ __forceinline__ Pos token_pos(const Plan &p, int jg) {
    Pos q;
    q.f = fast_div(jg, p.hw_m, p.hw_s);
    const int rem = jg - q.f * p.Hg * p.Wg;
    q.h = fast_div(rem, p.wg_m, p.wg_s);
    q.w = rem - q.h * p.Wg;
    return q;
}

// Where the records of feature group m sit in the table.
struct GroupRec {
    int base, stride, axis;
};

__device__ __forceinline__ GroupRec group_rec(const Plan &p, int m) {
    return GroupRec{p.hc_base[m], p.hc_stride[m], p.hc_axis[m]};
}

__device__ __forceinline__ float4 tab_rec(const uint8_t *tab, const GroupRec &g, const Pos &q) {
    const int pos = g.axis == 0 ? q.f : (g.axis == 1 ? q.h : q.w);
    return *reinterpret_cast<const float4 *>(tab + g.base + pos * g.stride);
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

__global__ void __launch_bounds__(kThreads, 1)
rope_reduce_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   float *__restrict__ partials, const Plan p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *tab = smem + kRTabOff;
    float *zbuf = reinterpret_cast<float *>(smem + kRZOff);
    uint64_t *raw_full = reinterpret_cast<uint64_t *>(smem + kRBarOff);
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
            mbar_init(&raw_empty[s], 1);
        }
        for (int o = 0; o < kROp; ++o) {
            mbar_init(&op_full[o], kNXf);
            mbar_init(&op_empty[o], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kNEpi);
            mbar_init(&z_full[a], kNXf);
            mbar_init(&z_empty[a], kNEpi);
        }
        mbar_init(drain, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    build_table(tab, p, threadIdx.x, kThreads);
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kRTmemCols);
        tmem_relinquish();
    }
    if (warp == kWarpTma && lane == 0) {
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
    int issued = 0;

    if (warp == kWarpTma) {
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
                    const int s = i % kRRaw;
                    if (!mbar_wait(&raw_empty[s], ((uint32_t)(i / kRRaw) & 1u) ^ 1u, abort_word, &g_rope_wait_flag,
                                   1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *stg = smem + s * kRStage;
                    const int row = sg.n * p.L + sg.tok0 + 32 * st;
                    const int c0 = sg.g * 128;
                    mbar_arrive_expect_tx(&raw_full[s], kRStage);
                    tma_load_3d(stg, &tm_k, &raw_full[s], c0, row, sg.b);
                    tma_load_3d(stg + kBox, &tm_k, &raw_full[s], c0 + 64, row, sg.b);
                    tma_load_3d(stg + 2 * kBox, &tm_v, &raw_full[s], c0, row, sg.b);
                    tma_load_3d(stg + 3 * kBox, &tm_v, &raw_full[s], c0 + 64, row, sg.b);
                    issued = i + 1;
                }
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, 128, 1, 1);
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
                    const uint32_t hi = smem_u32(smem + kROpOff + o * kRStage);
                    const uint32_t va = smem_u32(smem + s * kRStage + 2 * kBox);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        // MN-major, 128-byte swizzle: the two 64-feature boxes are the
                        // MN atoms (kBox apart), 8-token groups 1024 B apart
                        const uint64_t dh = smem_desc(hi + kk * 2048, kBox, 1024, kLayoutSw128);
                        const uint64_t dl = smem_desc(hi + 2 * kBox + kk * 2048, kBox, 1024, kLayoutSw128);
                        const uint64_t dv = smem_desc(va + kk * 2048, kBox, 1024, kLayoutSw128);
                        mma_bf16(d, dh, dv, idesc, (st > 0 || kk > 0) ? 1u : 0u);
                        mma_bf16(d, dl, dv, idesc, 1u);
                    }
                    mma_commit(&op_empty[o]);
                    mma_commit(&raw_empty[s]);   // v is read from the raw stage
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
        // reads TMEM lanes 32q.. = key features of head 4g + q
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
            const float z = zbuf[a * 128 + q * 32 + lane];
            tc_fence_before();
            mbar_arrive(&acc_empty[a]);
            mbar_arrive(&z_empty[a]);
            const int h = 4 * sg.g + q;
            float *dst = partials + ((((size_t)sg.b * p.H + h) * p.nb + sg.n) * p.skP + sg.slot) * kKVZ;
            float4 *drow = reinterpret_cast<float4 *>(dst + lane * kD);
#pragma unroll
            for (int j = 0; j < 8; ++j) drow[j] = make_float4(kv[4 * j], kv[4 * j + 1], kv[4 * j + 2], kv[4 * j + 3]);
            dst[kD * kD + lane] = z;
        }
    } else {
        // ------------------------------------------------ transform: one token row
        // (lane) per stage, feature chunk j of head hl (box 0) and of head 2 + hl
        // (box 1): the same 8 features, so one position and one pair of records
        const int wt = threadIdx.x - kXf0;
        const int j = (wt >> 5) & 3, hl = wt >> 7;
        const int r = lane;
        const int chunk = (((4 * hl + j) ^ (r & 7)) << 4) + r * 128;   // byte offset inside a box
        const GroupRec g0 = group_rec(p, 2 * j), g1 = group_rec(p, 2 * j + 1);
        Feat8 zs[2];
#pragma unroll
        for (int bx = 0; bx < 2; ++bx) zs[bx].e0 = zs[bx].o0 = zs[bx].e1 = zs[bx].o1 = make_float2(0.f, 0.f);
        UnitWalk w;
        w.start(S, x_begin);
        bool ok = true;
        int i = 0, sidx = 0;
        for (long long x = x_begin; x < x_end; x = w.end, ++sidx) {
            w.to(S, x);
            const Seg sg = seg_of(w, x);
            const int nst = (sg.tok1 - sg.tok0 + 31) / 32;
            for (int st = 0; st < nst; ++st, ++i) {
                const int s = i % kRRaw, o = i % kROp;
                if (ok && !mbar_wait(&raw_full[s], (uint32_t)(i / kRRaw) & 1u, abort_word, &g_rope_wait_flag, 6))
                    ok = false;
                if (ok && !mbar_wait(&op_empty[o], ((uint32_t)(i / kROp) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 7))
                    ok = false;
                const int tb = sg.tok0 + 32 * st + r;   // token of this row inside the block
                const uint8_t *raw = smem + s * kRStage;
                uint8_t *op = smem + kROpOff + o * kRStage;
                if (ok && tb < sg.tok1) {
                    const Pos pq = token_pos(p, sg.n * p.L + tb);
                    const float4 t0 = tab_rec(tab, g0, pq);
                    const float4 t1 = tab_rec(tab, g1, pq);
#pragma unroll
                    for (int bx = 0; bx < 2; ++bx) {
                        const uint4 xv = *reinterpret_cast<const uint4 *>(raw + bx * kBox + chunk);
                        uint4 hi, lo;
                        Feat8 f;
                        rope_chunk(xv, t0, t1, hi, lo, f);
                        zs[bx].e0 = fadd2(zs[bx].e0, f.e0);
                        zs[bx].o0 = fadd2(zs[bx].o0, f.o0);
                        zs[bx].e1 = fadd2(zs[bx].e1, f.e1);
                        zs[bx].o1 = fadd2(zs[bx].o1, f.o1);
                        *reinterpret_cast<uint4 *>(op + bx * kBox + chunk) = hi;
                        *reinterpret_cast<uint4 *>(op + 2 * kBox + bx * kBox + chunk) = lo;
                    }
                } else {
                    // rows past the segment contribute nothing
                    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int bx = 0; bx < 2; ++bx) {
                        *reinterpret_cast<uint4 *>(op + bx * kBox + chunk) = zero;
                        *reinterpret_cast<uint4 *>(op + 2 * kBox + bx * kBox + chunk) = zero;
                    }
                }
                // the generic writes of this stage before the tensor cores read it
                fence_proxy_async_smem();
                mbar_arrive(&op_full[o]);
            }
            // the segment's z: sum this thread's 16 features over the 32 rows
            float zv[16];
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
                const Feat8 &f = zs[bx];
                float *t = zv + 8 * bx;
                t[0] = f.e0.x; t[1] = f.o0.x; t[2] = f.e0.y; t[3] = f.o0.y;
                t[4] = f.e1.x; t[5] = f.o1.x; t[6] = f.e1.y; t[7] = f.o1.y;
                zs[bx].e0 = zs[bx].o0 = zs[bx].e1 = zs[bx].o1 = make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) zv[k] += __shfl_xor_sync(0xffffffffu, zv[k], off);
            const int a = sidx & 1;
            if (ok && !mbar_wait(&z_empty[a], ((uint32_t)(sidx >> 1) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 8))
                ok = false;
            if (lane == 0) {
#pragma unroll
                for (int bx = 0; bx < 2; ++bx) {
                    float4 *zz = reinterpret_cast<float4 *>(zbuf + a * 128 + (2 * bx + hl) * 32 + 8 * j);
                    zz[0] = make_float4(zv[8 * bx], zv[8 * bx + 1], zv[8 * bx + 2], zv[8 * bx + 3]);
                    zz[1] = make_float4(zv[8 * bx + 4], zv[8 * bx + 5], zv[8 * bx + 6], zv[8 * bx + 7]);
                }
            }
            __syncwarp();
            mbar_arrive(&z_full[a]);
        }
    }

    // teardown: nothing may still write this CTA's shared memory or TMEM
    if (warp == kWarpTma && lane == 0 && *abort_word) {
        for (int i = issued - kRRaw < 0 ? 0 : issued - kRRaw; i < issued; ++i)
            final_wait(&raw_full[i % kRRaw], (uint32_t)(i / kRRaw) & 1u);
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

__global__ void __launch_bounds__(kThreads, 1)
rope_apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
                  __nv_bfloat16 *__restrict__ out, const uint8_t *__restrict__ bop, const float *__restrict__ seff,
                  const Plan p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *tab = smem + kATabOff;
    uint8_t *bops = smem + kABopOff;
    float *den_s = reinterpret_cast<float *>(smem + kADenOff);
    uint64_t *raw_full = reinterpret_cast<uint64_t *>(smem + kABarOff);
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
            mbar_init(&raw_empty[s], kNXf);
        }
        for (int o = 0; o < kAOp; ++o) {
            mbar_init(&op_full[o], kNXf);
            mbar_init(&op_empty[o], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kNEpi);
            mbar_init(&den_full[a], kNXf);
            mbar_init(&den_empty[a], kNEpi);
            mbar_init(&bop_full[a], 1);
            mbar_init(&bop_empty[a], 1);
        }
        mbar_init(drain, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    build_table(tab, p, threadIdx.x, kThreads);
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kATmemCols);
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
    int issued = 0, bops_issued = 0;

    if (warp == kWarpTma) {
        if (lane == 0) {
            auto load_q = [&](const UnitWalk &w, long long x, int i) {
                const int s = i % kARaw;
                const int row = w.n * p.L + (int)(x - w.first) * 128;
                mbar_arrive_expect_tx(&raw_full[s], kATile);
                tma_load_3d(smem + s * kATile, &tm_q, &raw_full[s], w.u * 64, row, w.b);
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
            // started: the first tiles are fetched while the combine still runs
            const int pre = ntiles < kARaw ? ntiles : kARaw;
            UnitWalk w;
            w.start(S, x_begin);
            for (int i = 0; i < pre; ++i) {
                w.to(S, x_begin + i);
                load_q(w, x_begin + i, i);
            }
            pdl_wait();   // the packed operand and Z_eff are written by the combine
            w.start(S, x_begin);
            int kb = 0;
            for (int i = 0; i < ntiles; ++i) {
                const long long x = x_begin + i;
                if (w.to(S, x) || i == 0) {
                    if (!load_bop(w, kb++)) break;
                }
                if (i < pre) continue;
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
                const uint32_t qa = smem_u32(smem + kAOpOff + o * 2 * kATile);
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
                            // A: K-major, 128-byte swizzle; head hh is the 64-byte half of
                            // each 128-byte row, 16 features = 32 bytes per step
                            const uint64_t da =
                                smem_desc(qa + apart * kATile + hh * 64 + kk * 32, 16, 1024, kLayoutSw128);
                            // B: K-major, no swizzle, core matrices 128 B apart along K,
                            // 8-row groups 512 B apart; 16 features = 256 bytes per step
                            const uint64_t db =
                                smem_desc(ba + hh * 4096 + bpart * 2048 + kk * 256, 128, 512, kLayoutNone);
                            mma_bf16(d, da, db, idesc, (prod | kk) ? 1u : 0u);
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
    } else if (warp >= 6) {
        // ------------------------------------------------ transform: token row r of
        // the tile, the 4 feature chunks of head hh
        const int wt = threadIdx.x - kXf0;
        const int hh = wt >> 7, r = wt & 127;
        float2 ze[4][2], zo[4][2];   // Z_eff of head hh: chunk j, pairs (a, b) / (c, d), even / odd features
        UnitWalk w;
        w.start(S, x_begin);
        bool ok = true;
        int kb = -1;
        for (int i = 0; i < ntiles; ++i) {
            const long long x = x_begin + i;
            if (w.to(S, x) || i == 0) {
                ++kb;
                if (ok && !mbar_wait(&bop_full[kb & 1], (uint32_t)(kb >> 1) & 1u, abort_word, &g_rope_wait_flag, 16))
                    ok = false;
                const float4 *zsrc = reinterpret_cast<const float4 *>(bops + (kb & 1) * kABopBytes + 8192 + hh * 128);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 u0 = zsrc[2 * j], u1 = zsrc[2 * j + 1];   // features 8j .. 8j + 7
                    ze[j][0] = make_float2(u0.x, u0.z);
                    zo[j][0] = make_float2(u0.y, u0.w);
                    ze[j][1] = make_float2(u1.x, u1.z);
                    zo[j][1] = make_float2(u1.y, u1.w);
                }
            }
            const int s = i % kARaw, o = i % kAOp, a = i & 1;
            const int Ln = w.n < p.nb - 1 ? p.L : Llast;
            const int row0 = (int)(x - w.first) * 128;
            const bool valid = r < Ln - row0;
            if (ok && !mbar_wait(&raw_full[s], (uint32_t)(i / kARaw) & 1u, abort_word, &g_rope_wait_flag, 17)) ok = false;
            uint4 xq[4];
            const uint8_t *raw = smem + s * kATile + r * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                xq[j] = (ok && valid) ? *reinterpret_cast<const uint4 *>(raw + (((4 * hh + j) ^ (r & 7)) << 4))
                                      : make_uint4(0u, 0u, 0u, 0u);
            // the raw stage may be refilled as soon as every thread has read it:
            // order these generic reads before the async proxy's refill
            fence_proxy_async_smem();
            mbar_arrive(&raw_empty[s]);
            if (ok && !mbar_wait(&op_empty[o], ((uint32_t)(i / kAOp) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 18))
                ok = false;
            if (ok && !mbar_wait(&den_empty[a], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_word, &g_rope_wait_flag, 19))
                ok = false;
            uint8_t *op = smem + kAOpOff + o * 2 * kATile + r * 128;
            float2 den = make_float2(0.f, 0.f);
            if (ok && valid) {
                const Pos pq = token_pos(p, w.n * p.L + row0 + r);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 t0 = tab_rec(tab, group_rec(p, 2 * j), pq);
                    const float4 t1 = tab_rec(tab, group_rec(p, 2 * j + 1), pq);
                    uint4 hi, lo;
                    Feat8 f;
                    rope_chunk(xq[j], t0, t1, hi, lo, f);
                    // the denominator takes the unrotated phi(q)
                    den = ffma2(f.e0, ze[j][0], den);
                    den = ffma2(f.o0, zo[j][0], den);
                    den = ffma2(f.e1, ze[j][1], den);
                    den = ffma2(f.o1, zo[j][1], den);
                    const int pc = ((4 * hh + j) ^ (r & 7)) << 4;
                    *reinterpret_cast<uint4 *>(op + pc) = hi;
                    *reinterpret_cast<uint4 *>(op + kATile + pc) = lo;
                }
            } else {
                const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int pc = ((4 * hh + j) ^ (r & 7)) << 4;
                    *reinterpret_cast<uint4 *>(op + pc) = zero;
                    *reinterpret_cast<uint4 *>(op + kATile + pc) = zero;
                }
            }
            den_s[a * 256 + hh * 128 + r] = den.x + den.y;
            fence_proxy_async_smem();
            mbar_arrive(&op_full[o]);
            mbar_arrive(&den_full[a]);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int q = warp & 3;
        const int r = 32 * q + lane;               // token row of this thread in a tile
        uint8_t *sb = smem + kAStgOff + q * kBox;  // this warp's staging box
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
            float num0[32], num1[32], den0 = 0.f, den1 = 0.f;
            if (got) {
                tc_fence_after();
                const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 64);
                tmem_ld32(base, num0);
                tmem_ld32(base + 32, num1);
                tmem_wait_ld();
                den0 = den_s[a * 256 + r];
                den1 = den_s[a * 256 + 128 + r];
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[a]);
            mbar_arrive(&den_empty[a]);
            if (!got) continue;

            const int Ln = w.n < p.nb - 1 ? p.L : Llast;
            const int row0 = (int)(x - w.first) * 128;
            const int blk0 = w.n * p.L;                // first token of the block in the call
            const int wrow0 = blk0 + row0 + 32 * q;    // first row of this warp
            const float2 inv0 = make_float2(1.0f / (den0 + p.eps), 1.0f / (den0 + p.eps));
            const float2 inv1 = make_float2(1.0f / (den1 + p.eps), 1.0f / (den1 + p.eps));
            // TMA store of the warp's 32 rows unless they run into the next block
            // (rows past the end of the tensor are clipped by TMA)
            const bool boxed = row0 + 32 * q + 32 <= Ln || blk0 + Ln == p.N;
            if (boxed) {
                if (lane == 0) bulk_wait_read<0>();   // the last store from this box has read it
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c) {          // logical 16-byte chunk c: head c / 4
                    const float *v = c < 4 ? num0 : num1;
                    const float2 inv = c < 4 ? inv0 : inv1;
                    const int f0 = 8 * (c & 3);
                    const float2 y0 = fmul2(make_float2(v[f0], v[f0 + 1]), inv);
                    const float2 y1 = fmul2(make_float2(v[f0 + 2], v[f0 + 3]), inv);
                    const float2 y2 = fmul2(make_float2(v[f0 + 4], v[f0 + 5]), inv);
                    const float2 y3 = fmul2(make_float2(v[f0 + 6], v[f0 + 7]), inv);
                    const int pc = c ^ (lane & 7);     // 128-byte swizzle (row % 8 == lane % 8)
                    *reinterpret_cast<uint4 *>(sb + lane * 128 + pc * 16) =
                        make_uint4(pack_bf2(y0.x, y0.y), pack_bf2(y1.x, y1.y), pack_bf2(y2.x, y2.y),
                                   pack_bf2(y3.x, y3.y));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&tm_out, sb, w.u * 64, wrow0, w.b);
                    bulk_commit();
                }
            } else if (row0 + r < Ln) {
                // a short last tile of a block that is not the last of the tensor:
                // the rows after the block belong to the next block
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float *v = hh ? num1 : num0;
                    const float2 inv = hh ? inv1 : inv0;
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        out + (((size_t)w.b * p.N + blk0 + row0 + r) * p.H + 2 * w.u + hh) * kD);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 y0 = fmul2(make_float2(v[8 * c], v[8 * c + 1]), inv);
                        const float2 y1 = fmul2(make_float2(v[8 * c + 2], v[8 * c + 3]), inv);
                        const float2 y2 = fmul2(make_float2(v[8 * c + 4], v[8 * c + 5]), inv);
                        const float2 y3 = fmul2(make_float2(v[8 * c + 6], v[8 * c + 7]), inv);
                        dst[c] = make_uint4(pack_bf2(y0.x, y0.y), pack_bf2(y1.x, y1.y), pack_bf2(y2.x, y2.y),
                                            pack_bf2(y3.x, y3.y));
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    if (warp == kWarpTma && lane == 0 && *abort_word) {
        for (int kb = bops_issued - 2 < 0 ? 0 : bops_issued - 2; kb < bops_issued; ++kb)
            final_wait(&bop_full[kb & 1], (uint32_t)(kb >> 1) & 1u);
        for (int i = issued - kARaw < 0 ? 0 : issued - kARaw; i < issued; ++i)
            final_wait(&raw_full[i % kARaw], (uint32_t)(i / kARaw) & 1u);
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
        ok = set_smem((const void *)rope_reduce_kernel, kRSmem) && set_smem((const void *)rope_apply_kernel, kASmem);
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
    CUtensorMap mk, mv;
    if (!make_bf16_map(&mk, k, p.B, p.N, p.H, 32) || !make_bf16_map(&mv, v, p.B, p.N, p.H, 32)) return -1;
    return launch_pdl(rope_reduce_kernel, (unsigned)p.skr.C, kThreads, kRSmem, s, mk, mv, partials, p) ? 1 : -1;
}

int launch_apply_rope_tc(const void *q, void *out, const void *bop, const float *seff, const Plan &p,
                         cudaStream_t s) {
    if (!smem_ready() || !tc_rope_fits(p)) return -1;
    CUtensorMap mq, mo;
    if (!make_bf16_map(&mq, q, p.B, p.N, p.H, 128) || !make_bf16_map(&mo, out, p.B, p.N, p.H, 32)) return -1;
    return launch_pdl(rope_apply_kernel, (unsigned)p.ska.C, kThreads, kASmem, s, mq, mo,
                      static_cast<__nv_bfloat16 *>(out), static_cast<const uint8_t *>(bop), seff, p)
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
