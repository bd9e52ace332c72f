// k_bwd_tc.cu -- key side of the backward pass on the tensor cores.
//
// With G_m = sum_{n >= m} [dS_n | dZ_n] (the suffix sums of the state
// gradients, k_bwd.cu) and token t of block m (no RoPE):
//   dv_t = G_m^T phi(k_t)             (per head: D[t][c] = sum_a phi(K)[t][a] G[a][c])
//   dk_t = 1[k_t > 0] (G_m v_t + Gz_m) (per head: D[t][a] = sum_c V[t][c] G[a][c])
// Both are the shape of the forward apply: a 128-token tile of 2 heads as the
// A operand (K-major, 128-byte swizzle, as TMA lands it) against a packed
// 32 x 32 operand per head, G or G^T as a bf16 hi and a lo part accumulated in
// the same TMEM columns (G to ~16 bits).  The derivative of the recurrence the
// pages give ("Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı",
// section "Sabit Bellekli KV önbelleğe alma mekanizması"), for training.
//
// With RoPE (R the numerator rotation of each token, sd114.wiki SANA-Video
// summary, section "两大核心技术突破", item 1):
//   dv_t = G_m^T R phi(k_t),  dk_t = 1[k_t > 0] (R^T (G_m v_t) + Gz_m).
// The transform warps rotate phi(k) and split it into a bf16 hi part (in
// place of the k tile) and a lo part (a second tile), so dv takes three
// products (hi G_hi, hi G_lo, lo G_hi); the dk epilogue applies R^T to each
// head's 32 values of G_m v_t before adding Gz and the ReLU mask.
//
// Warp roles: 0 TMA (k and v tiles, prefetched before the dependency wait,
// then the packed operands), 1 TMEM + MMAs, 6..9 ReLU (and RoPE) on the k tile
// in shared memory and its sign bits, 2..5 epilogue (TMEM -> dk, dv, TMA
// stores).  Every wait is bounded; a wait that gives up raises the device
// flag.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "la_internal.cuh"
#include "la_rope.cuh"
#include "la_sm100.cuh"

namespace la {

using namespace sm100;

namespace {

// Raised by a bounded wait of this file's kernel that gave up (0x100 | where);
// read by la_device_status through read_and_clear_bwd_k_flag.
__device__ unsigned int g_wait_flag = 0;

constexpr int kKTThreads = 320;
constexpr int kKTWarpTma = 0, kKTWarpMma = 1, kKTXform0 = 192, kKTWork = 128;
constexpr int kKTTile = 128 * 128;             // [128 rows][64 bf16]: 2 heads of k (or v)
constexpr int kKTStages = 2;
constexpr int kKTStage = 2 * kKTTile;          // k tile, v tile
constexpr int kKTWarpStg = 32 * 128;           // one epilogue warp's staging box
constexpr int kKTOpsBytes = 2 * 4 * kGopBytes;  // 2 heads x (G hi, G lo, G^T hi, G^T lo)
constexpr int kKTMaskBytes = 2 * 128 * 8;       // [acc buffer][row][logical chunk] sign bytes
constexpr int kKTNumBars = 3 * kKTStages + 2 + 2 + 2 + 3;   // ring, acc_full, acc_empty, mask_ready, ops, dep, drain
constexpr int kKTTabBytes = 8192;              // RoPE: the call's cos/sin table
// Shared memory; with RoPE the lo parts of the rotated k tiles and the table
// are added (one CTA per SM then, two without).
template <bool ROPE>
struct KT {
    static constexpr int kLoOff = kKTStages * kKTStage;
    static constexpr int kStgOff = kLoOff + (ROPE ? kKTStages * kKTTile : 0);
    static constexpr int kOpsOff = kStgOff + 4 * kKTWarpStg;
    static constexpr int kMaskOff = kOpsOff + kKTOpsBytes;
    static constexpr int kGzOff = kMaskOff + kKTMaskBytes;
    static constexpr int kTabOff = kGzOff + 2 * kD * 4;
    static constexpr int kBarOff = kTabOff + (ROPE ? kKTTabBytes : 0);
    static constexpr int kSmem = kBarOff + kKTNumBars * 8 + 16 + 1024;
    static_assert(kSmem <= (ROPE ? 232448 : 232448 / 2), "key-side shared memory");
};
constexpr uint32_t kKTTmemCols = 256;           // 2 buffers x [dv h0 | dv h1 | dpk h0 | dpk h1]

template <bool ROPE>
__global__ void __launch_bounds__(kKTThreads, ROPE ? 1 : 2)
bwd_k_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv, const float *__restrict__ G,
                const uint8_t *__restrict__ gop, const Plan p) {
    using C = KT<ROPE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stg = smem + C::kStgOff;
    uint8_t *ops = smem + C::kOpsOff;
    uint8_t *mask8 = smem + C::kMaskOff;
    uint8_t *tab = smem + C::kTabOff;
    float *gz = reinterpret_cast<float *>(smem + C::kGzOff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *xform_done = full + kKTStages;
    uint64_t *empty = xform_done + kKTStages;
    uint64_t *acc_full = empty + kKTStages;     // [2]
    uint64_t *acc_empty = acc_full + 2;         // [2]
    uint64_t *mask_ready = acc_empty + 2;       // [2]
    uint64_t *ops_full = mask_ready + 2;
    uint64_t *dep_ready = ops_full + 1;
    uint64_t *drain = dep_ready + 1;
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
    pdl_trigger();
    if (ta1 <= ta0) return;
    const int ntiles = (int)((ta1 - ta0 + 127) / 128);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKTStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xform_done[s], kKTWork);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kKTWork);
            mbar_init(&mask_ready[a], kKTWork);
        }
        mbar_init(ops_full, 1);
        mbar_init(dep_ready, 1);
        mbar_init(drain, 1);
        *abort_word = 0;
        fence_barrier_init();
    }
    if (warp == kKTWarpMma) {
        tmem_alloc(tmem_slot, kKTTmemCols);
        tmem_relinquish();
    }
    if (warp == kKTWarpTma && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_dk);
        prefetch_tmap(&tm_dv);
    }
    if constexpr (ROPE) build_table(tab, p, threadIdx.x, kKTThreads);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0;
    bool ops_issued = false;

    if (warp == kKTWarpTma) {
        if (lane == 0) {
            // k and v are inputs of the call: their first tiles come in while the
            // previous kernel (the suffix sums) still runs
            const int pre = ntiles < kKTStages ? ntiles : kKTStages;
            for (int i = 0; i < pre; ++i) {
                mbar_arrive_expect_tx(&full[i], kKTStage);
                tma_load_3d(smem + i * kKTStage, &tm_k, &full[i], hp * 64, (int)(ta0 + 128LL * i), b);
                tma_load_3d(smem + i * kKTStage + kKTTile, &tm_v, &full[i], hp * 64, (int)(ta0 + 128LL * i), b);
                issued = i + 1;
            }
            pdl_wait();
            mbar_arrive(dep_ready);
            mbar_arrive_expect_tx(ops_full, kKTOpsBytes);
            for (int hh = 0; hh < 2; ++hh) {
                const size_t src = (((size_t)b * p.H + 2 * hp + hh) * p.nb + n) * 4 * (size_t)kGopBytes;
                bulk_load(ops + hh * 4 * kGopBytes, gop + src, 4 * kGopBytes, ops_full);
            }
            ops_issued = true;
            for (int i = pre; i < ntiles; ++i) {
                const int s = i % kKTStages;
                const uint32_t ph = (uint32_t)(i / kKTStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, &g_wait_flag, 51)) break;
                mbar_arrive_expect_tx(&full[s], kKTStage);
                tma_load_3d(smem + s * kKTStage, &tm_k, &full[s], hp * 64, (int)(ta0 + 128LL * i), b);
                tma_load_3d(smem + s * kKTStage + kKTTile, &tm_v, &full[s], hp * 64, (int)(ta0 + 128LL * i), b);
                issued = i + 1;
            }
        }
    } else if (warp == kKTWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, kD, 0, 0);
            const uint32_t oaddr = smem_u32(ops);
            if (mbar_wait(ops_full, 0, abort_word, &g_wait_flag, 52)) {
                for (int i = 0; i < ntiles; ++i) {
                    const int s = i % kKTStages;
                    const uint32_t ph = (uint32_t)(i / kKTStages) & 1u;
                    const int ab = i & 1;
                    const uint32_t aph = (uint32_t)(i >> 1) & 1u;
                    if (!mbar_wait(&xform_done[s], ph, abort_word, &g_wait_flag, 53)) break;
                    if (!mbar_wait(&acc_empty[ab], aph ^ 1u, abort_word, &g_wait_flag, 54)) break;
                    tc_fence_after();
                    const uint32_t kaddr = smem_u32(smem + s * kKTStage), vaddr = kaddr + kKTTile;
                    const uint32_t loaddr = smem_u32(smem + C::kLoOff + s * kKTTile);   // RoPE: R phi(K) lo
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                        for (int which = 0; which < 2; ++which) {   // 0: dv from phi(K) and G; 1: dpk from V and G^T
                            const uint32_t d = tmem + ab * 128 + which * 64 + hh * kD;
                            // products (A part, B part): (hi, hi), (hi, lo), and with RoPE for dv
                            // (lo, hi): A = R phi(K) is then a hi and a lo tile
                            const int nprod = (ROPE && which == 0) ? 3 : 2;
#pragma unroll
                            for (int prod = 0; prod < 3; ++prod) {
                                if (prod >= nprod) break;
                                const int apart = prod == 2 ? 1 : 0, part = prod == 1 ? 1 : 0;
                                const uint32_t abase = (which ? vaddr : (apart ? loaddr : kaddr)) + hh * 64;
#pragma unroll
                                for (int kk = 0; kk < 2; ++kk) {
                                    // A: K-major, 128-byte swizzle, head hh = 64-byte half of a row;
                                    // B: K-major, no swizzle, 128 B along K, 512 B per 8 rows
                                    const uint64_t da = smem_desc(abase + kk * 32, 16, 1024, kLayoutSw128);
                                    const uint64_t db = smem_desc(oaddr + (hh * 4 + which * 2 + part) * kGopBytes + kk * 256,
                                                                  128, 512, kLayoutNone);
                                    mma_bf16(d, da, db, idesc, (prod | kk) ? 1u : 0u);
                                }
                            }
                        }
                    }
                    mma_commit(&empty[s]);
                    mma_commit(&acc_full[ab]);
                }
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------ ReLU on the k tile, sign bytes
        const int tt = threadIdx.x - kKTXform0;
        // RoPE: this thread's chunks are all logical chunk L (the same 8 features of
        // one head) of rows tt / 8 + 16 j, so two table groups serve all of them
        const int Lc = (tt & 7) ^ ((tt >> 3) & 7);
        const GroupRec gr0 = group_rec(p, 2 * (Lc & 3)), gr1 = group_rec(p, 2 * (Lc & 3) + 1);
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % kKTStages;
            const uint32_t ph = (uint32_t)(i / kKTStages) & 1u;
            const int ab = i & 1;
            const uint32_t aph = (uint32_t)(i >> 1) & 1u;
            if (ok && !mbar_wait(&full[s], ph, abort_word, &g_wait_flag, 55)) ok = false;
            // the sign bytes of buffer ab are free once the epilogue of tile i-2 read them
            if (ok && !mbar_wait(&acc_empty[ab], aph ^ 1u, abort_word, &g_wait_flag, 56)) ok = false;
            uint8_t *kt = smem + s * kKTStage;
            uint8_t *lot = smem + C::kLoOff + s * kKTTile;
            Pos pq{};
            if constexpr (ROPE) pq = token_pos(p, (int)(ta0 + 128LL * i + (tt >> 3)));
            if (ok) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int u = tt + 128 * j;
                    const int row = u >> 3, L = (u & 7) ^ (row & 7);   // logical chunk: head L/4, features 8(L%4)..
                    uint4 *ptr = reinterpret_cast<uint4 *>(kt + (size_t)u * 16);
                    const uint4 x = *ptr;
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                    uint32_t bits = 0;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        // bf16 > 0: sign bit clear and not zero
                        bits |= (((w[m] & 0x8000u) == 0u && (w[m] & 0x7FFFu) != 0u) ? 1u : 0u) << (2 * m);
                        bits |= (((w[m] & 0x80000000u) == 0u && (w[m] & 0x7FFF0000u) != 0u) ? 1u : 0u) << (2 * m + 1);
                    }
                    mask8[ab * 1024 + row * 8 + L] = (uint8_t)bits;
                    if constexpr (ROPE) {
                        // rows past the tensor (TMA's zero fill) get zero hi and lo, and
                        // no table lookup at a position past the call's frames
                        uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
                        if (ta0 + 128LL * i + row < p.N) {
                            Feat8 f;
                            rope_chunk(x, tab_rec(tab, gr0, pq), tab_rec(tab, gr1, pq), hi, lo, f);
                        }
                        *ptr = hi;
                        *reinterpret_cast<uint4 *>(lot + (size_t)u * 16) = lo;
                        pos_step(p, pq, 16);
                    } else {
                        *ptr = make_uint4(relu2(x.x), relu2(x.y), relu2(x.z), relu2(x.w));
                    }
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&xform_done[s]);
            mbar_arrive(&mask_ready[ab]);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int wt = threadIdx.x - 64;
        const int qd = warp & 3;
        const int r = 32 * qd + lane;   // token row of this thread in a tile
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        uint8_t *sb = stg + qd * kKTWarpStg;
        bool ok = mbar_wait(dep_ready, 0, abort_word, &g_wait_flag, 57);
        if (wt < 2 * kD)   // Gz of the 2 heads, from the suffix sums
            gz[wt] = ok ? __ldcg(G + (((size_t)b * p.H + 2 * hp + (wt >> 5)) * p.nb + n) * kKVZ + kD * kD + (wt & 31))
                        : 0.f;
        named_bar_sync(3, kKTWork);
        for (int i = 0; i < ntiles; ++i) {
            const int ab = i & 1;
            const uint32_t aph = (uint32_t)(i >> 1) & 1u;
            bool got = ok && mbar_wait(&acc_full[ab], aph, abort_word, &g_wait_flag, 58);
            got = got && mbar_wait(&mask_ready[ab], aph, abort_word, &g_wait_flag, 59);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
            uint2 mk = make_uint2(0u, 0u);
            if (got) mk = *reinterpret_cast<const uint2 *>(mask8 + ab * 1024 + r * 8);
            // sign bits of this row: byte L covers logical chunk L (head L/4, features 8(L%4)..)
            const uint32_t m0 = mk.x, m1 = mk.y;
            const long long row0 = ta0 + 128LL * i;
            const long long wrow0 = row0 + 32 * qd;
            // RoPE: this row's position (rows past the tensor take the last token's;
            // their results are not stored)
            Pos pr{};
            if constexpr (ROPE) pr = token_pos(p, (int)(row0 + r < p.N ? row0 + r : p.N - 1));
            const bool boxed = wrow0 + 32 <= ta1 || ta1 == p.N;
            const uint32_t base = tmem + lane_off + ab * 128;
            for (int which = 0; which < 2; ++which) {   // 0: dk (TMEM columns 64..127), 1: dv (0..63)
                if (boxed) {
                    if (lane == 0) bulk_wait_read<0>();   // the previous store from sb has read it
                    __syncwarp();
                }
                for (int hh = 0; hh < 2; ++hh) {          // one head at a time: 32 values live
                    float h[32];
                    if (got) {
                        tc_fence_after();
                        tmem_ld32(base + (which ? 0 : 64) + hh * kD, h);
                        tmem_wait_ld();
                        if (!which) {
                            const uint32_t m = hh ? m1 : m0;
                            if constexpr (ROPE) {
                                // d phi(k) = R^T d psi(k): pair (x0, x1) by its (cos, sin) to
                                // (x0 cos + x1 sin, x1 cos - x0 sin); group g holds features 4g .. 4g + 3
#pragma unroll
                                for (int g = 0; g < 8; ++g) {
                                    const float4 t = tab_rec(tab, group_rec(p, g), pr);
                                    const float a0 = h[4 * g], a1 = h[4 * g + 1], b0 = h[4 * g + 2], b1 = h[4 * g + 3];
                                    h[4 * g] = fmaf(a1, t.z, a0 * t.x);
                                    h[4 * g + 1] = fmaf(-a0, t.z, a1 * t.x);
                                    h[4 * g + 2] = fmaf(b1, t.w, b0 * t.y);
                                    h[4 * g + 3] = fmaf(-b0, t.w, b1 * t.y);
                                }
                            }
#pragma unroll
                            for (int a = 0; a < 32; ++a) h[a] = (m >> a) & 1u ? h[a] + gz[hh * kD + a] : 0.f;
                        }
                    }
                    if (which && hh == 1) {   // the TMEM buffer and its sign bytes are read
                        tc_fence_before();
                        mbar_arrive(&acc_empty[ab]);
                    }
                    if (!got) continue;
                    if (boxed) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {   // logical chunk 4 hh + c4 of the row
                            const int pc = (4 * hh + c4) ^ (lane & 7);   // 128-byte swizzle
                            *reinterpret_cast<uint4 *>(sb + lane * 128 + pc * 16) =
                                make_uint4(pack_bf2(h[8 * c4], h[8 * c4 + 1]), pack_bf2(h[8 * c4 + 2], h[8 * c4 + 3]),
                                           pack_bf2(h[8 * c4 + 4], h[8 * c4 + 5]),
                                           pack_bf2(h[8 * c4 + 6], h[8 * c4 + 7]));
                        }
                    } else if (row0 + r < ta1) {
                        uint4 *dst = reinterpret_cast<uint4 *>(
                            (which ? dv : dk) + (((size_t)b * p.N + row0 + r) * p.H + 2 * hp + hh) * kD);
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            dst[c4] = make_uint4(pack_bf2(h[8 * c4], h[8 * c4 + 1]), pack_bf2(h[8 * c4 + 2], h[8 * c4 + 3]),
                                                 pack_bf2(h[8 * c4 + 4], h[8 * c4 + 5]),
                                                 pack_bf2(h[8 * c4 + 6], h[8 * c4 + 7]));
                    }
                }
                if (boxed) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && ok) {
                        tma_store_3d(which ? &tm_dv : &tm_dk, sb, hp * 64, (int)wrow0, b);
                        bulk_commit();
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    // teardown: nothing may still write this CTA's shared memory or TMEM
    if (warp == kKTWarpTma && lane == 0 && *abort_word) {
        if (ops_issued) final_wait(ops_full, 0);
        for (int i = issued - kKTStages < 0 ? 0 : issued - kKTStages; i < issued; ++i)
            final_wait(&full[i % kKTStages], (uint32_t)(i / kKTStages) & 1u);
    }
    if (warp == kKTWarpMma && lane == 0 && *abort_word) {
        mma_commit(drain);
        final_wait(drain, 0);
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == kKTWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kKTTmemCols);
    }
}

}  // namespace

bool bwd_k_tc_available(const Plan &p) {
    return tc_available() && p.H % 4 == 0 && !p.f8 && (!p.rope || (p.tab_bytes > 0 && p.tab_bytes <= kKTTabBytes));
}

int launch_bwd_k_tc(const void *k, const void *v, const float *G, const void *gop, void *dk, void *dv,
                    const Plan &p, cudaStream_t s) {
    static std::once_flag once;
    static bool attr_ok = false;
    std::call_once(once, [] {
        attr_ok = set_smem((const void *)bwd_k_tc_kernel<false>, KT<false>::kSmem) &&
                  set_smem((const void *)bwd_k_tc_kernel<true>, KT<true>::kSmem);
    });
    if (!attr_ok) return -1;
    if (p.rope && !bwd_k_tc_available(p)) return -1;
    CUtensorMap mk, mv, mdk, mdv;
    if (!make_bf16_map(&mk, k, p.B, p.N, p.H, 128) || !make_bf16_map(&mv, v, p.B, p.N, p.H, 128) ||
        !make_bf16_map(&mdk, dk, p.B, p.N, p.H, 32) || !make_bf16_map(&mdv, dv, p.B, p.N, p.H, 32))
        return -1;
    const long long grid = (long long)p.B * p.nb * p.Pa * (p.H / 2);
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    __nv_bfloat16 *dk16 = static_cast<__nv_bfloat16 *>(dk), *dv16 = static_cast<__nv_bfloat16 *>(dv);
    const uint8_t *g8 = static_cast<const uint8_t *>(gop);
    const bool ok = p.rope ? launch_pdl(bwd_k_tc_kernel<true>, (unsigned)grid, kKTThreads, KT<true>::kSmem, s, mk, mv,
                                        mdk, mdv, dk16, dv16, G, g8, p)
                           : launch_pdl(bwd_k_tc_kernel<false>, (unsigned)grid, kKTThreads, KT<false>::kSmem, s, mk,
                                        mv, mdk, mdv, dk16, dv16, G, g8, p);
    return ok ? 1 : -1;
}

int read_and_clear_bwd_k_flag(unsigned *flag_out) {
    unsigned zero = 0;
    if (cudaMemcpyFromSymbol(flag_out, g_wait_flag, sizeof(unsigned)) != cudaSuccess) return -1;
    if (*flag_out && cudaMemcpyToSymbol(g_wait_flag, &zero, sizeof(unsigned)) != cudaSuccess) return -1;
    return 0;
}

}  // namespace la
