// la_rope.cuh -- device helpers of the 3D RoPE on phi(q), phi(k) shared by
// the tensor-core kernels (forward reduce and apply, key side of the
// backward): packed fp32x2 arithmetic, the ReLU'd features of a 16-byte chunk,
// the rotation of feature pairs with the split into a hi and a lo part, and
// the cos/sin table of a call (sd114.wiki SANA-Video summary, section
// "两大核心技术突破", item 1: RoPE for the spatio-temporal position of each
// latent token).
//
// Table: for each of the 8 groups of 4 features m, its two pairs 2m, 2m+1 at
// every position along the group's axis (frames of the call, rows, columns),
// one 16-byte record (cos a, cos b, sin a, sin b) each, at the byte offsets
// plan_rope_table puts in the Plan.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "la_internal.cuh"
#include "la_sm100.cuh"

namespace la {
namespace {

using namespace sm100;

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

// ReLU of one chunk of 8 bf16 (4 feature pairs) as fp32.
__device__ __forceinline__ Feat8 relu_unpack_bf16(uint4 x) {
    const uint32_t wa = relu2(x.x), wb = relu2(x.y), wc = relu2(x.z), wd = relu2(x.w);
    Feat8 f;
    f.e0 = make_float2(bf_lo(wa), bf_lo(wb));
    f.o0 = make_float2(bf_hi(wa), bf_hi(wb));
    f.e1 = make_float2(bf_lo(wc), bf_lo(wd));
    f.o1 = make_float2(bf_hi(wc), bf_hi(wd));
    return f;
}

__device__ __forceinline__ float2 f16x2_f32(uint32_t h) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
    const __half2 t = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&t);
}

// Rotate the 4 feature pairs (x0, x1) of a chunk by their (cos, sin) to
// (x0 cos - x1 sin, x0 sin + x1 cos) and split the rotated values into a hi
// part RN(y) and a lo part RN(y - hi), bf16 (H16 false) or f16 (H16 true).
// t0 = (cos a, cos b, sin a, sin b), t1 the same for pairs c, d.
template <bool H16>
__device__ __forceinline__ void rotate_split(const Feat8 &f, float4 t0, float4 t1, uint4 &hi, uint4 &lo) {
    const float2 c0 = make_float2(t0.x, t0.y), s0 = make_float2(t0.z, t0.w);
    const float2 c1 = make_float2(t1.x, t1.y), s1 = make_float2(t1.z, t1.w);
    const float2 ye0 = ffma2(f.o0, make_float2(-s0.x, -s0.y), fmul2(f.e0, c0));
    const float2 yo0 = ffma2(f.o0, c0, fmul2(f.e0, s0));
    const float2 ye1 = ffma2(f.o1, make_float2(-s1.x, -s1.y), fmul2(f.e1, c1));
    const float2 yo1 = ffma2(f.o1, c1, fmul2(f.e1, s1));
    if constexpr (!H16) {
        hi = make_uint4(pack_bf2(ye0.x, yo0.x), pack_bf2(ye0.y, yo0.y), pack_bf2(ye1.x, yo1.x),
                        pack_bf2(ye1.y, yo1.y));
        // y - hi is exact in fp32
        const float2 re0 = fsub2(ye0, make_float2(bf_lo(hi.x), bf_lo(hi.y)));
        const float2 ro0 = fsub2(yo0, make_float2(bf_hi(hi.x), bf_hi(hi.y)));
        const float2 re1 = fsub2(ye1, make_float2(bf_lo(hi.z), bf_lo(hi.w)));
        const float2 ro1 = fsub2(yo1, make_float2(bf_hi(hi.z), bf_hi(hi.w)));
        lo = make_uint4(pack_bf2(re0.x, ro0.x), pack_bf2(re0.y, ro0.y), pack_bf2(re1.x, ro1.x),
                        pack_bf2(re1.y, ro1.y));
    } else {
        hi = make_uint4(pack_f16x2(ye0.x, yo0.x), pack_f16x2(ye0.y, yo0.y), pack_f16x2(ye1.x, yo1.x),
                        pack_f16x2(ye1.y, yo1.y));
        const float2 h0 = f16x2_f32(hi.x), h1 = f16x2_f32(hi.y), h2 = f16x2_f32(hi.z), h3 = f16x2_f32(hi.w);
        const float2 re0 = fsub2(ye0, make_float2(h0.x, h1.x));
        const float2 ro0 = fsub2(yo0, make_float2(h0.y, h1.y));
        const float2 re1 = fsub2(ye1, make_float2(h2.x, h3.x));
        const float2 ro1 = fsub2(yo1, make_float2(h2.y, h3.y));
        lo = make_uint4(pack_f16x2(re0.x, ro0.x), pack_f16x2(re0.y, ro0.y), pack_f16x2(re1.x, ro1.x),
                        pack_f16x2(re1.y, ro1.y));
    }
}

// ReLU one chunk of 8 bf16, rotate and split into bf16 hi and lo parts; f
// receives phi(x).
__device__ __forceinline__ void rope_chunk(uint4 x, float4 t0, float4 t1, uint4 &hi, uint4 &lo, Feat8 &f) {
    f = relu_unpack_bf16(x);
    rotate_split<false>(f, t0, t1, hi, lo);
}

// The (cos, sin) records of every position of the call: for each of the 8
// groups of 4 features m, its two pairs 2m, 2m+1 at every position along the
// group's axis (frames of the call, rows, columns), at the byte offsets the
// host planned.
__device__ void build_table(uint8_t *tab, const Plan &p, int tid, int nthr) {
    // (unrolled: the plan's arrays are then read at fixed offsets of the
    // kernel parameters, never copied to local memory)
#pragma unroll
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

// The position d tokens further on (d >= 0): columns wrap into rows, rows
// into frames.
__device__ __forceinline__ void pos_step(const Plan &p, Pos &q, int d) {
    q.w += d;
    while (q.w >= p.Wg) {
        q.w -= p.Wg;
        if (++q.h == p.Hg) {
            q.h = 0;
            ++q.f;
        }
    }
}

// Where the records of feature group m sit in the table.
struct GroupRec {
    int base, stride, axis;
};

__device__ __forceinline__ GroupRec group_rec(const Plan &p, int m) {
    // select by an unrolled compare, so that the parameter arrays are never
    // indexed at run time (which would copy them to local memory)
    GroupRec g{0, 0, 0};
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (k == m) g = GroupRec{p.hc_base[k], p.hc_stride[k], p.hc_axis[k]};
    return g;
}

__device__ __forceinline__ float4 tab_rec(const uint8_t *tab, const GroupRec &g, const Pos &q) {
    const int pos = g.axis == 0 ? q.f : (g.axis == 1 ? q.h : q.w);
    return *reinterpret_cast<const float4 *>(tab + g.base + pos * g.stride);
}


}  // namespace
}  // namespace la
