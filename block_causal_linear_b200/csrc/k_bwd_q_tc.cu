// k_bwd_q_tc.cu -- query side of the backward pass on the tensor cores.
//
// Per (b, h) and token t of block n, with S_n, Z_n the state after block n
// (no RoPE):
//   num_t = phi(q_t) S_n, den_t = phi(q_t) . Z_n + eps            (M1, as the forward apply)
//   g_t = dout_t / den_t, c_t = -(dout_t . num_t) / den_t^2          (epilogue, CUDA cores)
//   dq_t = 1[q_t > 0] (S_n g_t + c_t Z_n)                             (M2: g S^T, then the epilogue)
//   dS_n += phi(q_t) g_t^T, dZ_n += c_t phi(q_t)                      (M3, M4: summed over the split)
// The derivative of the recurrence the pages give ("Nvidia, MIT ve diğerleri
// video yapay zeka devrimini başlattı", section "Sabit Bellekli KV önbelleğe
// alma mekanizması").
//
// One CTA per (b, 4-head group, block, token split), 128-token tiles.  The q
// tile (4 heads, two 64-feature TMA boxes, 128-byte swizzle) is the K-major A
// operand of M1 and the MN-major A operand of M3/M4, as TMA lands it (after
// ReLU in place).  g is written by the epilogue as a bf16 hi and a lo tile in
// the same layout: the K-major A operand of M2 and the MN-major B operand of
// M3.  c goes into a [16 rows][128 tokens] operand (rows 2h, 2h + 1: c hi and
// c lo of head h) so that M4 gives dZ of head h as the sum of two columns.  The state operands S, S^T
// are bf16 hi + lo (~16 bits).  All sums have one fixed order.
//
// Warp roles: 0 TMA, 1 TMEM + MMAs, 2..5 ReLU on the q tile and its sign
// bytes, then the dq epilogue one tile behind (M2 -> dq), 6..9 the g epilogue
// (M1 -> g, c; at the end dS, dZ).  c passes between the two epilogues in a
// double buffer.  Every
// wait is bounded; a wait that gives up raises the device flag.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "la_internal.cuh"
#include "la_sm100.cuh"

namespace la {

using namespace sm100;

namespace {

// Raised by a bounded wait of this file's kernel that gave up (0x100 | where);
// read by la_device_status through read_and_clear_bwd_q_flag.
__device__ unsigned int g_wait_flag = 0;

constexpr int kQTThreads = 320;
constexpr int kQTWarpTma = 0, kQTWarpMma = 1, kQTXform0 = 64, kQTEpi0 = 192, kQTWork = 128;
constexpr int kQTBox = 128 * 128;                    // [128 rows][64 bf16] = 16 KiB: 2 heads
constexpr int kQTTile = 2 * kQTBox;                  // 4 heads
constexpr int kQTStages = 2;
constexpr int kQTGOff = kQTStages * kQTTile;         // g hi tile, then g lo tile
constexpr int kQTCOff = kQTGOff + 2 * kQTTile;       // c operand: [16 rows][128 tokens] bf16
constexpr int kQTCBytes = 2 * 2048;
constexpr int kQTOpsOff = kQTCOff + kQTCBytes;       // per head: [S|Z|0] hi, lo; S^T hi, lo
constexpr int kQTOpsHead = 2 * kOpBytes + 2 * kStOpBytes;
constexpr int kQTStgOff = kQTOpsOff + 4 * kQTOpsHead;   // 4 epilogue warps x 2 boxes [32 rows][64 bf16]
constexpr int kQTZOff = kQTStgOff + 4 * 2 * 4096;       // Z_n of the 4 heads
constexpr int kQTCValOff = kQTZOff + 4 * kD * 4;        // c per row and head, fp32, [2 buffers][128][4]
constexpr int kQTMaskOff = kQTCValOff + 2 * 128 * 4 * 4;  // sign bytes [2 buffers][128 rows][16 logical chunks]
constexpr int kQTBarOff = kQTMaskOff + 2 * 128 * 16;
constexpr int kQTNumBars = 3 * kQTStages + 14;
constexpr int kQTSmem = kQTBarOff + kQTNumBars * 8 + 16 + 1024;
// TMEM columns
constexpr uint32_t kQTAcc1 = 0;      // num | den per head: 4 x 48
constexpr uint32_t kQTAcc2 = 192;    // S g per head: 4 x 32
constexpr uint32_t kQTAccS = 320;    // dS: 128 x 128 (4 diagonal 32 x 32 blocks used)
constexpr uint32_t kQTAccZ = 448;    // dZ: columns 0 (c hi) and 1 (c lo) of 16
constexpr uint32_t kQTTmemCols = 512;

// byte offset of (row n, token t) in the c operand: K-major, no swizzle, core
// matrices of 8 rows x 8 tokens, 128 B apart along the tokens, 2048 B per 8
// rows.  Rows 2h and 2h + 1 hold c hi and c lo of head h of the group.
__device__ __forceinline__ int c_offset(int n, int t) {
    return (n >> 3) * 2048 + (t >> 3) * 128 + (n & 7) * 16 + (t & 7) * 2;
}

__global__ void __launch_bounds__(kQTThreads, 1)
bwd_q_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_dq,
                const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ dout,
                __nv_bfloat16 *__restrict__ dq, const float *__restrict__ seff, const uint8_t *__restrict__ bop,
                const uint8_t *__restrict__ stop, float *__restrict__ bpart, const Plan p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *gtile = smem + kQTGOff;
    uint8_t *cop = smem + kQTCOff;
    uint8_t *ops = smem + kQTOpsOff;
    uint8_t *stg = smem + kQTStgOff;
    float *zs = reinterpret_cast<float *>(smem + kQTZOff);
    float *cval = reinterpret_cast<float *>(smem + kQTCValOff);
    uint8_t *mask8 = smem + kQTMaskOff;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQTBarOff);
    uint64_t *xform_done = full + kQTStages;
    uint64_t *empty = xform_done + kQTStages;
    uint64_t *acc1_full = empty + kQTStages;
    uint64_t *acc1_empty = acc1_full + 1;
    uint64_t *g_ready = acc1_empty + 1;
    uint64_t *g_free = g_ready + 1;
    uint64_t *acc2_full = g_free + 1;
    uint64_t *acc2_empty = acc2_full + 1;
    uint64_t *accS_full = acc2_empty + 1;
    uint64_t *ops_full = accS_full + 1;
    uint64_t *dep_ready = ops_full + 1;
    uint64_t *drain = dep_ready + 1;
    uint64_t *c_ready = drain + 1;             // [2] a tile's c values are written (g epilogue)
    uint64_t *c_free = c_ready + 2;            // [2] ... and read by the dq epilogue
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c_free + 2);
    volatile int *abort_word = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int G4 = p.H / 4;
    long long id = blockIdx.x;
    const int g = (int)(id % G4); id /= G4;
    const int sp = (int)(id % p.P); id /= p.P;
    const int n = (int)(id % p.nb); id /= p.nb;
    const int b = (int)id;
    const long long blk0 = (long long)n * p.L;
    const long long blk1 = blk0 + p.L < p.N ? blk0 + p.L : (long long)p.N;
    const long long t0 = blk0 + (long long)sp * p.chunk;
    const long long t1 = t0 + p.chunk < blk1 ? t0 + p.chunk : blk1;
    const int ntiles = t1 > t0 ? (int)((t1 - t0 + 127) / 128) : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (ntiles == 0) {   // a split past the end of a short last block: its sums are zero
        pdl_wait();
        for (int e = threadIdx.x; e < 4 * kKVZ; e += kQTThreads)
            bpart[((((size_t)b * p.H + 4 * g + e / kKVZ) * p.nb + n) * p.P + sp) * kKVZ + e % kKVZ] = 0.f;
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < kQTStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xform_done[s], kQTWork);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc1_full, 1);
        mbar_init(acc1_empty, kQTWork);
        mbar_init(g_ready, kQTWork);
        mbar_init(g_free, 1);
        mbar_init(acc2_full, 1);
        mbar_init(acc2_empty, kQTWork);
        mbar_init(accS_full, 1);
        mbar_init(ops_full, 1);
        mbar_init(dep_ready, 1);
        mbar_init(drain, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&c_ready[a], kQTWork);
            mbar_init(&c_free[a], kQTWork);
        }
        *abort_word = 0;
        fence_barrier_init();
    }
    // rows 8..15 of the c operand stay zero
    for (int i = threadIdx.x; i < kQTCBytes / 16; i += kQTThreads)
        reinterpret_cast<uint4 *>(cop)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == kQTWarpMma) {
        tmem_alloc(tmem_slot, kQTTmemCols);
        tmem_relinquish();
    }
    if (warp == kQTWarpTma && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_dq);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0;
    bool ops_issued = false;

    if (warp == kQTWarpTma) {
        if (lane == 0) {
            // q is an input of the call: its first tiles come in before the
            // dependency on the state combine resolves
            const int pre = ntiles < kQTStages ? ntiles : kQTStages;
            for (int i = 0; i < pre; ++i) {
                mbar_arrive_expect_tx(&full[i], kQTTile);
                const int row = (int)(t0 + 128LL * i);
                tma_load_3d(smem + i * kQTTile, &tm_q, &full[i], g * 128, row, b);
                tma_load_3d(smem + i * kQTTile + kQTBox, &tm_q, &full[i], g * 128 + 64, row, b);
                issued = i + 1;
            }
            pdl_wait();
            mbar_arrive(dep_ready);
            mbar_arrive_expect_tx(ops_full, 4 * kQTOpsHead);
            for (int hh = 0; hh < 4; ++hh) {
                const size_t bh = (size_t)b * p.H + 4 * g + hh;
                bulk_load(ops + hh * kQTOpsHead, bop + (bh * p.nb + n) * 2 * kOpBytes, 2 * kOpBytes, ops_full);
                bulk_load(ops + hh * kQTOpsHead + 2 * kOpBytes, stop + (bh * p.nb + n) * 2 * kStOpBytes,
                          2 * kStOpBytes, ops_full);
            }
            ops_issued = true;
            for (int i = pre; i < ntiles; ++i) {
                const int s = i % kQTStages;
                const uint32_t ph = (uint32_t)(i / kQTStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, &g_wait_flag, 61)) break;
                mbar_arrive_expect_tx(&full[s], kQTTile);
                const int row = (int)(t0 + 128LL * i);
                tma_load_3d(smem + s * kQTTile, &tm_q, &full[s], g * 128, row, b);
                tma_load_3d(smem + s * kQTTile + kQTBox, &tm_q, &full[s], g * 128 + 64, row, b);
                issued = i + 1;
            }
        }
    } else if (warp == kQTWarpMma) {
        if (lane == 0) {
            const uint32_t id_m1 = idesc_bf16(128, kOpRows, 0, 0);     // phi(Q) x [S|Z|0]
            const uint32_t id_m2 = idesc_bf16(128, kD, 0, 0);          // g x S^T
            const uint32_t id_m3 = idesc_bf16(128, 128, 1, 1);         // phi(Q)^T x g
            const uint32_t id_m4 = idesc_bf16(128, 16, 1, 0);          // phi(Q)^T x [c hi | c lo | 0]
            const uint32_t oaddr = smem_u32(ops), gaddr = smem_u32(gtile), caddr = smem_u32(cop);
            bool ok = mbar_wait(ops_full, 0, abort_word, &g_wait_flag, 62);
            for (int i = 0; i < ntiles && ok; ++i) {
                const int s = i % kQTStages;
                const uint32_t ph = (uint32_t)(i / kQTStages) & 1u;
                const uint32_t tph = (uint32_t)i & 1u;
                if (!mbar_wait(&xform_done[s], ph, abort_word, &g_wait_flag, 63)) break;
                if (!mbar_wait(acc1_empty, tph ^ 1u, abort_word, &g_wait_flag, 64)) break;
                tc_fence_after();
                const uint32_t qaddr = smem_u32(smem + s * kQTTile);
                // M1: per head, num | den from the packed [S | Z | 0] (hi, lo)
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint64_t da = smem_desc(qaddr + (hh >> 1) * kQTBox + (hh & 1) * 64 + kk * 32, 16,
                                                          1024, kLayoutSw128);
                            const uint64_t db = smem_desc(oaddr + hh * kQTOpsHead + part * kOpBytes + kk * 256, 128,
                                                          512, kLayoutNone);
                            mma_bf16(tmem + kQTAcc1 + hh * kOpRows, da, db, id_m1, (part | kk) ? 1u : 0u);
                        }
                }
                mma_commit(acc1_full);
                // M2..M4 once the epilogue has turned M1 into g and c
                if (!mbar_wait(g_ready, tph, abort_word, &g_wait_flag, 65)) break;
                if (!mbar_wait(acc2_empty, tph ^ 1u, abort_word, &g_wait_flag, 66)) break;
                tc_fence_after();
                // M2: per head, g S^T as g_hi.ST_hi + g_hi.ST_lo + g_lo.ST_hi
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
#pragma unroll
                    for (int prod = 0; prod < 3; ++prod) {
                        const int gp = prod == 2 ? 1 : 0, sp2 = prod == 1 ? 1 : 0;
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint64_t da = smem_desc(gaddr + gp * kQTTile + (hh >> 1) * kQTBox + (hh & 1) * 64 +
                                                              kk * 32,
                                                          16, 1024, kLayoutSw128);
                            const uint64_t db = smem_desc(oaddr + hh * kQTOpsHead + 2 * kOpBytes + sp2 * kStOpBytes +
                                                              kk * 256,
                                                          128, 512, kLayoutNone);
                            mma_bf16(tmem + kQTAcc2 + hh * kD, da, db, id_m2, (prod | kk) ? 1u : 0u);
                        }
                    }
                }
                // M3, M4: over the tile's 128 tokens, 16 per MMA; MN-major, the two
                // 64-feature boxes kQTBox apart (LBO), 8-token groups 1024 B apart (SBO)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t da = smem_desc(qaddr + kk * 2048, kQTBox, 1024, kLayoutSw128);
#pragma unroll
                    for (int gp = 0; gp < 2; ++gp) {
                        const uint64_t db = smem_desc(gaddr + gp * kQTTile + kk * 2048, kQTBox, 1024, kLayoutSw128);
                        mma_bf16(tmem + kQTAccS, da, db, id_m3, (i > 0 || kk > 0 || gp > 0) ? 1u : 0u);
                    }
                    const uint64_t dc = smem_desc(caddr + kk * 256, 128, 2048, kLayoutNone);
                    mma_bf16(tmem + kQTAccZ, da, dc, id_m4, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&empty[s]);   // the q tile is read
                mma_commit(g_free);      // g and c are read
                mma_commit(acc2_full);
            }
            mma_commit(accS_full);
        }
    } else if (warp < 6) {
        // ------------------------------------------------ warps 2..5: ReLU on the q tile and its sign
        // bytes for tile i + 1, then the dq epilogue of tile i (one tile behind warps 6..9)
        const int tt = threadIdx.x - kQTXform0;
        const int qd = warp & 3;                // TMEM lane quarter
        const int r = 32 * qd + lane;           // token row of this thread in a tile
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        uint8_t *sb = stg + qd * 2 * 4096;      // this warp's two staging boxes
        bool ok = mbar_wait(dep_ready, 0, abort_word, &g_wait_flag, 69);
        {   // Z_n of the 4 heads
            const size_t bh = (size_t)b * p.H + 4 * g + (tt >> 5);
            zs[tt] = ok ? __ldcg(seff + (bh * p.nb + n) * kKVZ + kD * kD + (tt & 31)) : 0.f;
        }
        auto transform = [&](int i) {
            const int s = i % kQTStages;
            const uint32_t ph = (uint32_t)(i / kQTStages) & 1u;
            if (ok && !mbar_wait(&full[s], ph, abort_word, &g_wait_flag, 67)) ok = false;
            uint8_t *qt = smem + s * kQTTile;
            uint8_t *mk = mask8 + (i & 1) * 2048;
            const long long row0 = t0 + 128LL * i;
            if (ok) {
#pragma unroll 4
                for (int j = 0; j < 16; ++j) {            // 2048 chunks of 16 bytes, 16 per thread
                    const int u = tt + 128 * j;
                    const int bx = u >> 10, row = (u >> 3) & 127;
                    const int L = (u & 7) ^ (row & 7);     // logical chunk within the box: head 2bx + L/4
                    uint4 *ptr = reinterpret_cast<uint4 *>(qt + (size_t)u * 16);
                    uint4 x = *ptr;
                    if (row0 + row >= t1) x = make_uint4(0u, 0u, 0u, 0u);   // rows past the split: nothing
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                    uint32_t bits = 0;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        bits |= (((w[m] & 0x8000u) == 0u && (w[m] & 0x7FFFu) != 0u) ? 1u : 0u) << (2 * m);
                        bits |= (((w[m] & 0x80000000u) == 0u && (w[m] & 0x7FFF0000u) != 0u) ? 1u : 0u) << (2 * m + 1);
                    }
                    mk[row * 16 + bx * 8 + L] = (uint8_t)bits;
                    *ptr = make_uint4(relu2(x.x), relu2(x.y), relu2(x.z), relu2(x.w));
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&xform_done[s]);
        };
        transform(0);
        for (int i = 0; i < ntiles; ++i) {
            // sign-byte buffer (i + 1) % 2 was last read by this group's dq epilogue of tile i - 1
            // (and every sign byte of tile i, and Z_n, is written)
            named_bar_sync(5, kQTWork);
            if (i + 1 < ntiles) transform(i + 1);
            // ---- E2: dq = mask (S g + c Z) from M2
            const int cb = i & 1;
            const uint32_t cph = (uint32_t)(i >> 1) & 1u;
            bool got2 = ok && mbar_wait(acc2_full, (uint32_t)i & 1u, abort_word, &g_wait_flag, 72);
            got2 = got2 && mbar_wait(&c_ready[cb], cph, abort_word, &g_wait_flag, 73);
            got2 = __all_sync(0xffffffffu, got2);
            if (!got2) ok = false;
            const long long row0 = t0 + 128LL * i;
            const long long t = row0 + r;
            const bool valid = t < t1;
            const long long wrow0 = row0 + 32 * qd;
            const bool boxed = wrow0 + 32 <= t1 || t1 == p.N;   // TMA clips rows >= N
            if (boxed) {
                if (lane == 0) bulk_wait_read<0>();   // the previous tile's stores have read sb
                __syncwarp();
            }
#pragma unroll 1
            for (int hh = 0; hh < 4; ++hh) {
                float pre[32];
                uint32_t m = 0;
                float cr = 0.f;
                if (got2) {
                    tc_fence_after();
                    tmem_ld32(tmem + lane_off + kQTAcc2 + hh * kD, pre);
                    tmem_wait_ld();
                    m = *reinterpret_cast<const uint32_t *>(mask8 + (i & 1) * 2048 + r * 16 + (hh >> 1) * 8 +
                                                            (hh & 1) * 4);
                    cr = cval[cb * 512 + r * 4 + hh];
                }
                if (hh == 3) {   // the M2 result and the c values are read
                    tc_fence_before();
                    mbar_arrive(acc2_empty);
                    mbar_arrive(&c_free[cb]);
                }
                if (!got2) continue;
#pragma unroll
                for (int a = 0; a < 32; ++a) pre[a] = (m >> a) & 1u ? fmaf(cr, zs[hh * kD + a], pre[a]) : 0.f;
                if (boxed) {
                    uint8_t *bx = sb + (hh >> 1) * 4096 + lane * 128;
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int pc = (4 * (hh & 1) + c4) ^ (lane & 7);   // 128-byte swizzle
                        *reinterpret_cast<uint4 *>(bx + pc * 16) =
                            make_uint4(pack_bf2(pre[8 * c4], pre[8 * c4 + 1]), pack_bf2(pre[8 * c4 + 2], pre[8 * c4 + 3]),
                                       pack_bf2(pre[8 * c4 + 4], pre[8 * c4 + 5]),
                                       pack_bf2(pre[8 * c4 + 6], pre[8 * c4 + 7]));
                    }
                } else if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(dq + (((size_t)b * p.N + t) * p.H + 4 * g + hh) * kD);
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        dst[c4] = make_uint4(pack_bf2(pre[8 * c4], pre[8 * c4 + 1]), pack_bf2(pre[8 * c4 + 2], pre[8 * c4 + 3]),
                                             pack_bf2(pre[8 * c4 + 4], pre[8 * c4 + 5]),
                                             pack_bf2(pre[8 * c4 + 6], pre[8 * c4 + 7]));
                }
            }
            if (boxed) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && ok) {
                    tma_store_3d(&tm_dq, sb, g * 128, (int)wrow0, b);
                    tma_store_3d(&tm_dq, sb + 4096, g * 128 + 64, (int)wrow0, b);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    } else {
        // ------------------------------------------------ epilogue warps 6..9: g and c from M1
        const int qd = warp & 3;                // TMEM lane quarter
        const int r = 32 * qd + lane;           // token row of this thread in a tile
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const uint32_t tph = (uint32_t)i & 1u;
            const int cb = i & 1;
            const long long row0 = t0 + 128LL * i;
            const long long t = row0 + r;
            const bool valid = t < t1;
            // dout of this token, 4 heads (256 bytes), loaded before the waits
            uint4 dv[16];
            {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    dout + (((size_t)b * p.N + (valid ? t : t0)) * p.H + 4 * g) * kD);
#pragma unroll
                for (int j = 0; j < 16; ++j) dv[j] = valid ? __ldg(src + j) : make_uint4(0u, 0u, 0u, 0u);
            }
            bool got = ok && mbar_wait(acc1_full, tph, abort_word, &g_wait_flag, 70);
            got = got && mbar_wait(g_free, tph ^ 1u, abort_word, &g_wait_flag, 71);   // M2..M4 of tile i-1 are done
            got = got && mbar_wait(&c_free[cb], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_word, &g_wait_flag, 75);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                float num[32], den = 0.f;
                if (got) {
                    tc_fence_after();
                    tmem_ld32(tmem + lane_off + kQTAcc1 + hh * kOpRows, num);
                    den = tmem_ld1(tmem + lane_off + kQTAcc1 + hh * kOpRows + kD);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) num[c] = 0.f;
                }
                if (hh == 3) {   // every head's M1 result is read
                    tc_fence_before();
                    mbar_arrive(acc1_empty);
                }
                float o[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 u = dv[4 * hh + j];
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        o[8 * j + 2 * m] = __uint_as_float(w[m] << 16);
                        o[8 * j + 2 * m + 1] = __uint_as_float(w[m] & 0xFFFF0000u);
                    }
                }
                const float inv = 1.0f / (den + p.eps);
                float dn = 0.f;
#pragma unroll
                for (int c = 0; c < 32; ++c) dn = fmaf(o[c], num[c], dn);
                const float cr = valid && got ? -dn * inv * inv : 0.f;
                // g hi and lo into the two g tiles: box hh/2, logical chunks 4 (hh%2) + c4
                uint8_t *gbox = gtile + (hh >> 1) * kQTBox + r * 128;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float g0 = valid && got ? o[8 * c4 + 2 * m] * inv : 0.f;
                        const float g1 = valid && got ? o[8 * c4 + 2 * m + 1] * inv : 0.f;
                        const __nv_bfloat162 hv = __floats2bfloat162_rn(g0, g1);
                        hi[m] = *reinterpret_cast<const uint32_t *>(&hv);
                        lo[m] = pack_bf2(g0 - __low2float(hv), g1 - __high2float(hv));
                    }
                    const int pc = (4 * (hh & 1) + c4) ^ (r & 7);
                    *reinterpret_cast<uint4 *>(gbox + pc * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(gbox + kQTTile + pc * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
                const __nv_bfloat16 ch = __float2bfloat16_rn(cr);
                *reinterpret_cast<__nv_bfloat16 *>(cop + c_offset(2 * hh, r)) = ch;
                *reinterpret_cast<__nv_bfloat16 *>(cop + c_offset(2 * hh + 1, r)) =
                    __float2bfloat16_rn(cr - __bfloat162float(ch));
                cval[cb * 512 + r * 4 + hh] = cr;
            }
            fence_proxy_async_smem();   // g and c are read by the tensor cores
            mbar_arrive(g_ready);
            mbar_arrive(&c_ready[cb]);
        }
        // ---- the split's [dS | dZ]: lane quarter qd = the key features of head 4g + qd
        bool gs = ok && mbar_wait(accS_full, 0, abort_word, &g_wait_flag, 74);
        gs = __all_sync(0xffffffffu, gs);
        if (gs) {
            tc_fence_after();
            float kv[32];
            tmem_ld32(tmem + lane_off + kQTAccS + 32 * qd, kv);
            const float z0 = tmem_ld1(tmem + lane_off + kQTAccZ + 2 * qd);
            const float z1 = tmem_ld1(tmem + lane_off + kQTAccZ + 2 * qd + 1);
            tmem_wait_ld();
            float *dst = bpart + ((((size_t)b * p.H + 4 * g + qd) * p.nb + n) * p.P + sp) * kKVZ;
            float4 *drow = reinterpret_cast<float4 *>(dst + lane * kD);
#pragma unroll
            for (int j = 0; j < 8; ++j) drow[j] = make_float4(kv[4 * j], kv[4 * j + 1], kv[4 * j + 2], kv[4 * j + 3]);
            dst[kD * kD + lane] = z0 + z1;
        }
        if (lane == 0) bulk_wait_all();
    }

    // teardown: nothing may still write this CTA's shared memory or TMEM
    if (warp == kQTWarpTma && lane == 0 && *abort_word) {
        if (ops_issued) final_wait(ops_full, 0);
        for (int i = issued - kQTStages < 0 ? 0 : issued - kQTStages; i < issued; ++i)
            final_wait(&full[i % kQTStages], (uint32_t)(i / kQTStages) & 1u);
    }
    if (warp == kQTWarpMma && lane == 0 && *abort_word) {
        mma_commit(drain);
        final_wait(drain, 0);
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == kQTWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kQTTmemCols);
    }
}

}  // namespace

bool bwd_q_tc_available(const Plan &p) { return tc_available() && p.H % 4 == 0 && !p.rope && !p.f8; }

// One CTA per SM (the kernel takes 512 TMEM columns and ~210 KiB of shared
// memory): the split plan aims at one wave of 148 CTAs.
void bwd_q_tc_plan(Plan &p) {
    const long long groups = (long long)p.B * (p.H / 4) * p.nb;
    long long want = 148 / groups;
    const long long maxw = (p.L + 127) / 128;
    if (want > maxw) want = maxw;
    if (want < 1) want = 1;
    long long chunk = (p.L + want - 1) / want;
    chunk = (chunk + 127) / 128 * 128;
    p.chunk = (int)chunk;
    p.P = (int)((p.L + chunk - 1) / chunk);
}

int launch_bwd_q_tc(const void *q, const void *dout, void *dq, const float *seff, const void *bop, const void *stop,
                    float *bpart, const Plan &p, cudaStream_t s) {
    static std::once_flag once;
    static bool attr_ok = false;
    std::call_once(once, [] { attr_ok = set_smem((const void *)bwd_q_tc_kernel, kQTSmem); });
    if (!attr_ok) return -1;
    CUtensorMap mq, mdq;
    if (!make_bf16_map(&mq, q, p.B, p.N, p.H, 128) || !make_bf16_map(&mdq, dq, p.B, p.N, p.H, 32)) return -1;
    const long long grid = (long long)p.B * (p.H / 4) * p.nb * p.P;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    return launch_pdl(bwd_q_tc_kernel, (unsigned)grid, kQTThreads, kQTSmem, s, mq, mdq,
                      static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(dout),
                      static_cast<__nv_bfloat16 *>(dq), seff, static_cast<const uint8_t *>(bop),
                      static_cast<const uint8_t *>(stop), bpart, p)
               ? 1
               : -1;
}

int read_and_clear_bwd_q_flag(unsigned *flag_out) {
    unsigned zero = 0;
    if (cudaMemcpyFromSymbol(flag_out, g_wait_flag, sizeof(unsigned)) != cudaSuccess) return -1;
    if (*flag_out && cudaMemcpyToSymbol(g_wait_flag, &zero, sizeof(unsigned)) != cudaSuccess) return -1;
    return 0;
}

}  // namespace la
