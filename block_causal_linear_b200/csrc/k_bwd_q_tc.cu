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
// c lo of head h) so that M4 gives dZ of head h as the sum of two columns.
// The state operands S, S^T are bf16 hi + lo (~16 bits).  All sums have one
// fixed order.
//
// The work of a tile is cut at its two 64-feature boxes (2 heads each): M1
// of box 0, the g epilogue of box 0 and the MMAs that read it (M2 of its heads,
// M3 against its g columns) run while the epilogue works on box 1, and M1 of
// the next tile is issued between them, so that the tensor cores and the
// epilogue overlap.
//
// Warp roles: 0 TMA, 1 TMEM + MMAs, 2..5 ReLU on the q tile and its sign
// bytes, 6..9 the g epilogue (M1 -> g, c; at the end dS, dZ), 10..13 the dq
// epilogue (M2 -> dq, staged for TMA stores).  c passes between the two
// epilogues in a double buffer, the sign bytes in a ring of four.  Every wait
// is bounded; a wait that gives up raises the device flag.
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

constexpr int kQTThreads = 448;
constexpr int kQTWarpTma = 0, kQTWarpMma = 1, kQTWork = 128;
constexpr int kQTXform0 = 64, kQTDq0 = 320;   // first thread of the transform and the dq warps
constexpr int kQTBox = 128 * 128;                    // [128 rows][64 bf16] = 16 KiB: 2 heads
constexpr int kQTTile = 2 * kQTBox;                  // 4 heads
constexpr int kQTStages = 2;
constexpr int kQTMaskBufs = 4;
constexpr int kQTGOff = kQTStages * kQTTile;         // g hi tile, then g lo tile
constexpr int kQTDoOff = kQTGOff + 2 * kQTTile;      // the dout tile, laid out as the q tile
constexpr int kQTCOff = kQTDoOff + kQTTile;          // c operand: [16 rows][128 tokens] bf16
constexpr int kQTCBytes = 2 * 2048;
constexpr int kQTOpsOff = kQTCOff + kQTCBytes;       // per head: [S|Z|0] hi, lo
constexpr int kQTOpsHead = 2 * kOpBytes;
constexpr int kQTStgOff = kQTOpsOff + 4 * kQTOpsHead;   // 4 dq warps x one box [32 rows][64 bf16]
constexpr int kQTAcOff = kQTStgOff + 4 * 4096;          // c as the K = 16 extension of M2's A: [128 tokens][16]
constexpr int kQTBcOff = kQTAcOff + 4096;               // Z_n as that extension of B, per head [32][16]
constexpr int kQTMaskOff = kQTBcOff + 4096;             // sign bytes [4 buffers][128 rows][16 logical chunks]
constexpr int kQTBarOff = kQTMaskOff + kQTMaskBufs * 128 * 16;
constexpr int kQTNumBars = 3 * kQTStages + 2 * kQTMaskBufs + 16;
constexpr int kQTSmem = kQTBarOff + kQTNumBars * 8 + 16 + 1024;
static_assert(kQTSmem <= 232448, "shared memory of the query-side kernel");
// TMEM columns
constexpr uint32_t kQTAcc1 = 0;      // num | den per head: 4 x 48 (box b: heads 2b, 2b + 1)
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

// The product c_t Z_n of dq is folded into M2 as one more K = 16 step per
// head.  Its A operand holds, per token t, the columns 3h, 3h + 1, 3h + 2 =
// c hi, c lo, c hi of head h (12..15 zero); the B operand of head h holds,
// per key feature f, the rows 3h, 3h + 1, 3h + 2 = Z hi, Z hi, Z lo (others
// zero), so the step adds (c hi + c lo) Z hi + c hi Z lo.  Both are K-major
// without swizzle: core matrices of 8 rows x 8 columns, the two column halves
// 128 B apart, 8-row groups 256 B apart.
__device__ __forceinline__ int ac_offset(int t, int k) {
    return (t >> 3) * 256 + (k >> 3) * 128 + (t & 7) * 16 + (k & 7) * 2;
}

__global__ void __launch_bounds__(kQTThreads, 1)
bwd_q_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dq, __nv_bfloat16 *__restrict__ dq,
                const float *__restrict__ seff, const uint8_t *__restrict__ bop, float *__restrict__ bpart,
                const Plan p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *gtile = smem + kQTGOff;
    uint8_t *cop = smem + kQTCOff;
    uint8_t *ops = smem + kQTOpsOff;
    uint8_t *stg = smem + kQTStgOff;
    uint8_t *dot = smem + kQTDoOff;
    uint8_t *acx = smem + kQTAcOff;
    uint8_t *bcx = smem + kQTBcOff;
    uint8_t *mask8 = smem + kQTMaskOff;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQTBarOff);
    uint64_t *xform_done = full + kQTStages;
    uint64_t *empty = xform_done + kQTStages;
    uint64_t *mask_ready = empty + kQTStages;      // [4] a tile's sign bytes are written
    uint64_t *mask_free = mask_ready + kQTMaskBufs; // [4] ... and read by the dq epilogue
    uint64_t *acc1_full = mask_free + kQTMaskBufs;  // [2] per box: M1 done
    uint64_t *acc1_empty = acc1_full + 2;           // [2] per box: the g epilogue has read it
    uint64_t *g_ready = acc1_empty + 2;             // [2] per box: g (and at box 1, c) written
    uint64_t *g_free = g_ready + 2;                 // M2, M3, M4 of a tile are done with g and c
    uint64_t *acc2_full = g_free + 1;
    uint64_t *acc2_empty = acc2_full + 1;
    uint64_t *bc_ready = acc2_empty + 1;            // the Z_n operand is written
    uint64_t *accS_full = bc_ready + 1;
    uint64_t *ops_full = accS_full + 1;
    uint64_t *dep_ready = ops_full + 1;
    uint64_t *drain = dep_ready + 1;
    uint64_t *dout_full = drain + 1;                // the dout tile is loaded
    uint64_t *dout_free = dout_full + 1;            // ... and read by the g epilogue
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dout_free + 1);
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
        for (int a = 0; a < kQTMaskBufs; ++a) {
            mbar_init(&mask_ready[a], kQTWork);
            mbar_init(&mask_free[a], kQTWork);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc1_full[a], 1);
            mbar_init(&acc1_empty[a], kQTWork);
            mbar_init(&g_ready[a], kQTWork);
        }
        mbar_init(g_free, 1);
        mbar_init(acc2_full, 1);
        mbar_init(acc2_empty, kQTWork);
        mbar_init(bc_ready, kQTWork);
        mbar_init(accS_full, 1);
        mbar_init(ops_full, 1);
        mbar_init(dep_ready, 1);
        mbar_init(drain, 1);
        mbar_init(dout_full, 1);
        mbar_init(dout_free, kQTWork);
        *abort_word = 0;
        fence_barrier_init();
    }
    // rows 8..15 of the c operand and columns 12..15 of its M2 form stay zero
    for (int i = threadIdx.x; i < kQTCBytes / 16; i += kQTThreads)
        reinterpret_cast<uint4 *>(cop)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < 4096 / 16; i += kQTThreads)
        reinterpret_cast<uint4 *>(acx)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == kQTWarpMma) {
        tmem_alloc(tmem_slot, kQTTmemCols);
        tmem_relinquish();
    }
    if (warp == kQTWarpTma && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_dq);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int issued = 0, do_issued = 0;
    bool ops_issued = false;

    if (warp == kQTWarpTma) {
        if (lane == 0) {
            auto load_q = [&](int i) {
                const int s = i % kQTStages;
                const int row = (int)(t0 + 128LL * i);
                mbar_arrive_expect_tx(&full[s], kQTTile);
                tma_load_3d(smem + s * kQTTile, &tm_q, &full[s], g * 128, row, b);
                tma_load_3d(smem + s * kQTTile + kQTBox, &tm_q, &full[s], g * 128 + 64, row, b);
                issued = i + 1;
            };
            auto load_dout = [&](int i) {
                const int row = (int)(t0 + 128LL * i);
                mbar_arrive_expect_tx(dout_full, kQTTile);
                tma_load_3d(dot, &tm_do, dout_full, g * 128, row, b);
                tma_load_3d(dot + kQTBox, &tm_do, dout_full, g * 128 + 64, row, b);
                do_issued = i + 1;
            };
            // q and dout are inputs of the call: their first tiles come in before
            // the dependency on the state combine resolves
            const int pre = ntiles < kQTStages ? ntiles : kQTStages;
            for (int i = 0; i < pre; ++i) load_q(i);
            load_dout(0);
            pdl_wait();
            mbar_arrive(dep_ready);
            mbar_arrive_expect_tx(ops_full, 4 * kQTOpsHead);
            for (int hh = 0; hh < 4; ++hh) {
                const size_t bh = (size_t)b * p.H + 4 * g + hh;
                bulk_load(ops + hh * kQTOpsHead, bop + (bh * p.nb + n) * 2 * kOpBytes, 2 * kOpBytes, ops_full);
            }
            ops_issued = true;
            // per tile: its q tile once a stage is free, then its dout tile once the
            // g epilogue has read the previous one (q first: it is needed earlier)
            for (int i = 1; i < ntiles; ++i) {
                if (i >= pre) {
                    const uint32_t ph = (uint32_t)(i / kQTStages) & 1u;
                    if (!mbar_wait(&empty[i % kQTStages], ph ^ 1u, abort_word, &g_wait_flag, 61)) break;
                    load_q(i);
                }
                if (!mbar_wait(dout_free, (uint32_t)(i - 1) & 1u, abort_word, &g_wait_flag, 60)) break;
                load_dout(i);
            }
        }
    } else if (warp == kQTWarpMma) {
        if (lane == 0) {
            const uint32_t id_m1 = idesc_bf16(128, kOpRows, 0, 0);     // phi(Q) x [S|Z|0]
            const uint32_t id_m2 = idesc_bf16(128, kD, 0, 1);          // g x S^T, S^T read MN-major
            const uint32_t id_m2c = idesc_bf16(128, kD, 0, 0);         // [c] x [Z], both K-major
            const uint32_t id_m3 = idesc_bf16(128, 128, 1, 1);         // phi(Q)^T x g
            const uint32_t id_m4 = idesc_bf16(128, 16, 1, 0);          // phi(Q)^T x [c hi | c lo | 0]
            const uint32_t oaddr = smem_u32(ops), gaddr = smem_u32(gtile), caddr = smem_u32(cop);
            const uint32_t acaddr = smem_u32(acx), bcaddr = smem_u32(bcx);
            // M1 of box bx (heads 2bx, 2bx + 1) of tile i: num | den from the packed [S | Z | 0] (hi, lo)
            auto m1 = [&](int i, int bx) {
                const uint32_t qaddr = smem_u32(smem + (i % kQTStages) * kQTTile) + bx * kQTBox;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int hh = 2 * bx + h2;
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint64_t da = smem_desc(qaddr + h2 * 64 + kk * 32, 16, 1024, kLayoutSw128);
                            const uint64_t db = smem_desc(oaddr + hh * kQTOpsHead + part * kOpBytes + kk * 256, 128,
                                                          512, kLayoutNone);
                            mma_bf16(tmem + kQTAcc1 + hh * kOpRows, da, db, id_m1, (part | kk) ? 1u : 0u);
                        }
                }
                mma_commit(&acc1_full[bx]);
            };
            // M2 of box bx: per head, g S^T as g_hi.ST_hi + g_hi.ST_lo + g_lo.ST_hi.  S^T is
            // the packed [S|Z|0] operand of M1 read MN-major: its value columns are
            // the K rows of S^T (8-row groups 512 B apart: LBO), its key features
            // the N columns (8-column chunks 128 B apart: SBO)
            auto m2 = [&](int bx) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int hh = 2 * bx + h2;
#pragma unroll
                    for (int prod = 0; prod < 3; ++prod) {
                        const int gp = prod == 2 ? 1 : 0, sp2 = prod == 1 ? 1 : 0;
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint64_t da = smem_desc(gaddr + gp * kQTTile + bx * kQTBox + h2 * 64 + kk * 32, 16,
                                                          1024, kLayoutSw128);
                            const uint64_t db = smem_desc(oaddr + hh * kQTOpsHead + sp2 * kOpBytes + kk * 1024, 512,
                                                          128, kLayoutNone);
                            mma_bf16(tmem + kQTAcc2 + hh * kD, da, db, id_m2, (prod | kk) ? 1u : 0u);
                        }
                    }
                    // + c_t Z_n: the K = 16 extension
                    mma_bf16(tmem + kQTAcc2 + hh * kD, smem_desc(acaddr, 128, 256, kLayoutNone),
                             smem_desc(bcaddr + hh * 1024, 128, 256, kLayoutNone), id_m2c, 1u);
                }
            };
            bool ok = mbar_wait(ops_full, 0, abort_word, &g_wait_flag, 62);
            ok = ok && mbar_wait(&xform_done[0], 0, abort_word, &g_wait_flag, 63);
            if (ok) {
                tc_fence_after();
                m1(0, 0);
                m1(0, 1);
            }
            ok = ok && mbar_wait(bc_ready, 0, abort_word, &g_wait_flag, 78);
            // per tile i: M2 of box 0, M1 of box 0 of tile i + 1, M2 of box 1 with M3 and
            // M4, M1 of box 1 of tile i + 1
            for (int i = 0; i < ntiles && ok; ++i) {
                const int s = i % kQTStages;
                const uint32_t tph = (uint32_t)i & 1u;
                const bool next = i + 1 < ntiles;
                if (!mbar_wait(&g_ready[0], tph, abort_word, &g_wait_flag, 65)) break;
                if (!mbar_wait(acc2_empty, tph ^ 1u, abort_word, &g_wait_flag, 66)) break;
                tc_fence_after();
                m2(0);
                if (next) {
                    const uint32_t ph1 = (uint32_t)((i + 1) / kQTStages) & 1u;
                    if (!mbar_wait(&xform_done[(i + 1) % kQTStages], ph1, abort_word, &g_wait_flag, 63)) break;
                    if (!mbar_wait(&acc1_empty[0], tph, abort_word, &g_wait_flag, 64)) break;
                    tc_fence_after();
                    m1(i + 1, 0);
                }
                if (!mbar_wait(&g_ready[1], tph, abort_word, &g_wait_flag, 67)) break;
                tc_fence_after();
                m2(1);
                // M3, M4: over the tile's 128 tokens, 16 per MMA; MN-major, the two
                // 64-feature boxes kQTBox apart (LBO), 8-token groups 1024 B apart (SBO)
                const uint32_t qaddr = smem_u32(smem + s * kQTTile);
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
                if (next) {
                    if (!mbar_wait(&acc1_empty[1], tph, abort_word, &g_wait_flag, 68)) break;
                    tc_fence_after();
                    m1(i + 1, 1);
                }
            }
            mma_commit(accS_full);
        }
    } else if (warp < 6) {
        // ------------------------------------------------ warps 2..5: ReLU on the q tile, its sign bytes
        const int tt = threadIdx.x - kQTXform0;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % kQTStages;
            const int mb = i % kQTMaskBufs;
            if (ok && !mbar_wait(&full[s], (uint32_t)(i / kQTStages) & 1u, abort_word, &g_wait_flag, 76)) ok = false;
            if (ok && !mbar_wait(&mask_free[mb], ((uint32_t)(i / kQTMaskBufs) & 1u) ^ 1u, abort_word, &g_wait_flag, 77))
                ok = false;
            uint8_t *qt = smem + s * kQTTile;
            uint8_t *mk = mask8 + mb * 2048;
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
            mbar_arrive(&mask_ready[mb]);
        }
    } else if (warp < 10) {
        // ------------------------------------------------ warps 6..9: the g epilogue, from M1
        const int qd = warp & 3;                // TMEM lane quarter
        const int r = 32 * qd + lane;           // token row of this thread in a tile
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const uint32_t tph = (uint32_t)i & 1u;
            const long long t = t0 + 128LL * i + r;
            const bool valid = t < t1;
#pragma unroll 1
            for (int bx = 0; bx < 2; ++bx) {
                bool got = ok && mbar_wait(&acc1_full[bx], tph, abort_word, &g_wait_flag, 70);
                if (bx == 0) {   // M2, M3, M4 of tile i - 1 are done with g and c; this tile's dout is in
                    got = got && mbar_wait(g_free, tph ^ 1u, abort_word, &g_wait_flag, 71);
                    got = got && mbar_wait(dout_full, tph, abort_word, &g_wait_flag, 75);
                }
                got = __all_sync(0xffffffffu, got);
                if (!got) ok = false;
                // this row's dout of the box's 2 heads (rows past the split are not used)
                uint4 cur[8];
                const uint8_t *drow = dot + bx * kQTBox + r * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) cur[j] = *reinterpret_cast<const uint4 *>(drow + ((j ^ (r & 7)) * 16));
                if (bx == 1) {
                    // the dout tile is read: order these generic loads before TMA
                    // (async proxy) refills the tile
                    fence_proxy_async_smem();
                    mbar_arrive(dout_free);
                }
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int hh = 2 * bx + h2;
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
                    if (h2 == 1) {   // both heads of the box are read
                        tc_fence_before();
                        mbar_arrive(&acc1_empty[bx]);
                    }
                    const float inv = 1.0f / (den + p.eps);
                    float dn = 0.f;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 u = cur[4 * h2 + j];
                        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            dn = fmaf(bf_lo(w[m]), num[8 * j + 2 * m], dn);
                            dn = fmaf(bf_hi(w[m]), num[8 * j + 2 * m + 1], dn);
                        }
                    }
                    const bool live = valid && got;
                    const float cr = live ? -dn * inv * inv : 0.f;
                    const float sc = live ? inv : 0.f;
                    // g hi and lo into the two g tiles: box bx, logical chunks 4 h2 + c4
                    uint8_t *gbox = gtile + bx * kQTBox + r * 128;
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const uint4 u = cur[4 * h2 + c4];
                        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const float g0 = bf_lo(w[m]) * sc;
                            const float g1 = bf_hi(w[m]) * sc;
                            const __nv_bfloat162 hv = __floats2bfloat162_rn(g0, g1);
                            hi[m] = *reinterpret_cast<const uint32_t *>(&hv);
                            lo[m] = pack_bf2(g0 - __low2float(hv), g1 - __high2float(hv));
                        }
                        const int pc = (4 * h2 + c4) ^ (r & 7);
                        *reinterpret_cast<uint4 *>(gbox + pc * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4 *>(gbox + kQTTile + pc * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                    const __nv_bfloat16 ch = __float2bfloat16_rn(cr);
                    *reinterpret_cast<__nv_bfloat16 *>(cop + c_offset(2 * hh, r)) = ch;
                    *reinterpret_cast<__nv_bfloat16 *>(cop + c_offset(2 * hh + 1, r)) =
                        __float2bfloat16_rn(cr - __bfloat162float(ch));
                    *reinterpret_cast<__nv_bfloat16 *>(acx + ac_offset(r, 3 * hh)) = ch;
                    *reinterpret_cast<__nv_bfloat16 *>(acx + ac_offset(r, 3 * hh + 1)) =
                        __float2bfloat16_rn(cr - __bfloat162float(ch));
                    *reinterpret_cast<__nv_bfloat16 *>(acx + ac_offset(r, 3 * hh + 2)) = ch;
                }
                fence_proxy_async_smem();   // the box's g (and its c) is read by the tensor cores
                mbar_arrive(&g_ready[bx]);
            }
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
    } else {
        // ------------------------------------------------ warps 10..13: the dq epilogue, from M2
        const int tt = threadIdx.x - kQTDq0;
        const int qd = warp & 3;                // TMEM lane quarter
        const int r = 32 * qd + lane;           // token row of this thread in a tile
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        bool ok = mbar_wait(dep_ready, 0, abort_word, &g_wait_flag, 69);
        {   // the Z_n operand of the folded c Z step: head tt / 32, key feature tt % 32
            const int h = tt >> 5, f = tt & 31;
            const size_t bh = (size_t)b * p.H + 4 * g + h;
            const float z = ok ? __ldcg(seff + (bh * p.nb + n) * kKVZ + kD * kD + f) : 0.f;
            const __nv_bfloat16 zh = __float2bfloat16_rn(z);
            const __nv_bfloat16 zl = __float2bfloat16_rn(z - __bfloat162float(zh));
            uint4 row[2];
            __nv_bfloat16 *e = reinterpret_cast<__nv_bfloat16 *>(row);
#pragma unroll
            for (int k = 0; k < 16; ++k)
                e[k] = (k == 3 * h || k == 3 * h + 1) ? zh : (k == 3 * h + 2 ? zl : __float2bfloat16_rn(0.f));
            *reinterpret_cast<uint4 *>(bcx + h * 1024 + ac_offset(f, 0)) = row[0];
            *reinterpret_cast<uint4 *>(bcx + h * 1024 + ac_offset(f, 8)) = row[1];
            fence_proxy_async_smem();
            mbar_arrive(bc_ready);
        }
        for (int i = 0; i < ntiles; ++i) {
            const int mb = i % kQTMaskBufs;
            bool got = ok && mbar_wait(acc2_full, (uint32_t)i & 1u, abort_word, &g_wait_flag, 72);
            got = got && mbar_wait(&mask_ready[mb], (uint32_t)(i / kQTMaskBufs) & 1u, abort_word, &g_wait_flag, 73);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
            const long long row0 = t0 + 128LL * i;
            const long long t = row0 + r;
            const bool valid = t < t1;
            const long long wrow0 = row0 + 32 * qd;
            const bool boxed = wrow0 + 32 <= t1 || t1 == p.N;   // TMA clips rows >= N
            uint8_t *sb = stg + qd * 4096;                     // this warp's staging box
            if (boxed) {
                if (lane == 0) bulk_wait_read<0>();   // the previous tile's stores have read sb
                __syncwarp();
            }
#pragma unroll 1
            for (int hh = 0; hh < 4; ++hh) {
                if (hh == 2 && boxed) {   // heads 0, 1 go out; the box then takes heads 2, 3
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (ok) {
                            tma_store_3d(&tm_dq, sb, g * 128, (int)wrow0, b);
                            bulk_commit();
                        }
                        bulk_wait_read<0>();
                    }
                    __syncwarp();
                }
                float pre[32];
                uint32_t m = 0;
                if (got) {
                    tc_fence_after();
                    tmem_ld32(tmem + lane_off + kQTAcc2 + hh * kD, pre);
                    tmem_wait_ld();
                    m = *reinterpret_cast<const uint32_t *>(mask8 + mb * 2048 + r * 16 + (hh >> 1) * 8 + (hh & 1) * 4);
                }
                if (hh == 3) {   // the M2 result and the sign bytes are read
                    tc_fence_before();
                    mbar_arrive(acc2_empty);
                    mbar_arrive(&mask_free[mb]);
                }
                if (!got) continue;
#pragma unroll
                for (int a = 0; a < 32; ++a) pre[a] = (m >> a) & 1u ? pre[a] : 0.f;
                if (boxed) {
                    uint8_t *bx = sb + lane * 128;
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
                    tma_store_3d(&tm_dq, sb, g * 128 + 64, (int)wrow0, b);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    // teardown: nothing may still write this CTA's shared memory or TMEM
    if (warp == kQTWarpTma && lane == 0 && *abort_word) {
        if (ops_issued) final_wait(ops_full, 0);
        for (int i = issued - kQTStages < 0 ? 0 : issued - kQTStages; i < issued; ++i)
            final_wait(&full[i % kQTStages], (uint32_t)(i / kQTStages) & 1u);
        if (do_issued > 0) final_wait(dout_full, (uint32_t)(do_issued - 1) & 1u);
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

// One CTA per SM (the kernel takes 512 TMEM columns and ~218 KiB of shared
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

int launch_bwd_q_tc(const void *q, const void *dout, void *dq, const float *seff, const void *bop, float *bpart,
                    const Plan &p, cudaStream_t s) {
    static std::once_flag once;
    static bool attr_ok = false;
    std::call_once(once, [] { attr_ok = set_smem((const void *)bwd_q_tc_kernel, kQTSmem); });
    if (!attr_ok) return -1;
    CUtensorMap mq, mdo, mdq;
    if (!make_bf16_map(&mq, q, p.B, p.N, p.H, 128) || !make_bf16_map(&mdo, dout, p.B, p.N, p.H, 128) ||
        !make_bf16_map(&mdq, dq, p.B, p.N, p.H, 32))
        return -1;
    const long long grid = (long long)p.B * (p.H / 4) * p.nb * p.P;
    if (grid <= 0 || grid > 0x7fffffffLL) return -1;
    return launch_pdl(bwd_q_tc_kernel, (unsigned)grid, kQTThreads, kQTSmem, s, mq, mdo, mdq,
                      static_cast<__nv_bfloat16 *>(dq), seff, static_cast<const uint8_t *>(bop), bpart, p)
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
