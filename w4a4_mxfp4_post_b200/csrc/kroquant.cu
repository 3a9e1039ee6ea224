// kroquant.cu -- sm_100a kernels and the C ABI (include/kroquant.h) of the
// KroQuant online activation quantizer and its two baselines.
//
// Operation ("KroQuant: Kronecker-Structured Block Transforms for Efficient
// Post-Training Quantization of Diffusion Transformers", arXiv 2607.21446,
// abstract; section 3.2, Eq. (4) as summarised by the Pith review): for every
// 32-channel block of every bf16 token row, y = (G1 (x) ... (x) G5) x, then
// MXFP4 (OCP MX v1.0, section 6.3): E8M0 scale 2^(floor(log2 amax) - 2),
// E2M1 codes by round-to-nearest-even with saturation.
//
// Design: the path is a pure stream (2 B read, 0.53 B written per element) so
// every kernel reads each activation byte once with 16-byte loads and writes
// codes and scales once; the Kronecker product is never materialised -- its
// five 2x2 factors are applied as radix-2 butterflies on values held in
// registers.  One thread owns one 32-element block, so no shuffles are needed;
// consecutive threads own consecutive blocks of the flattened [M*d/32] block
// array, so a warp reads 2 KB contiguous and writes 512 B of codes and 32 B of
// scales contiguous.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cmath>
#include <cstring>
#include <utility>

#include "kroquant.h"

namespace {

constexpr int kBlk = 32;           // MX block size == Kronecker block size
constexpr int kThreads = 256;      // threads per CTA for the streaming kernels

// ---------------------------------------------------------------------------
// error reporting
// ---------------------------------------------------------------------------
thread_local char tl_err[512] = "";

int fail(int status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(tl_err, sizeof tl_err, fmt, ap);
    va_end(ap);
    return status;
}

int ok()
{
    tl_err[0] = '\0';
    return KQ_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------

// bf16 -> fp32 is exact: a bf16 is the upper half of a binary32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack32(const uint4 (&raw)[4], float (&v)[32])
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            v[8 * q + 2 * h] = bf16_lo(w[h]);
            v[8 * q + 2 * h + 1] = bf16_hi(w[h]);
        }
    }
}

// One radix-2 Kronecker stage: the 2x2 factor F acts on in-block index bit
// BIT, i.e. on every pair (i, i | 1<<BIT) with bit BIT of i clear.
template <int BIT>
__device__ __forceinline__ void kron_stage(float (&v)[32], float f00, float f01, float f10, float f11)
{
#pragma unroll
    for (int i = 0; i < kBlk; ++i) {
        if (i & (1 << BIT)) continue;
        const float lo = v[i];
        const float hi = v[i | (1 << BIT)];
        v[i] = fmaf(f01, hi, f00 * lo);
        v[i | (1 << BIT)] = fmaf(f11, hi, f10 * lo);
    }
}

// y = (G1 (x) G2 (x) G3 (x) G4 (x) G5) v.  G1 (f[0..3]) acts on bit 4, G5
// (f[16..19]) on bit 0.  The five stages act on different index bits and
// therefore commute; they run from bit 0 up.
__device__ __forceinline__ void kron_apply(float (&v)[32], const float (&f)[20])
{
    kron_stage<0>(v, f[16], f[17], f[18], f[19]);
    kron_stage<1>(v, f[12], f[13], f[14], f[15]);
    kron_stage<2>(v, f[8], f[9], f[10], f[11]);
    kron_stage<3>(v, f[4], f[5], f[6], f[7]);
    kron_stage<4>(v, f[0], f[1], f[2], f[3]);
}

// E8M0 byte of a block from amax >= 0: e = floor(log2 amax) - 2 clamped to
// [-127, 127] is, for a normal amax, (exponent field - 127) - 2, so the byte
// e + 127 is (exponent field - 2); subnormal amax and 0 clamp to byte 0, the
// largest finite amax gives 252.
__device__ __forceinline__ uint32_t e8m0_byte(float amax)
{
    const uint32_t ef = __float_as_uint(amax) >> 23;
    return ef > 2u ? ef - 2u : 0u;
}

// 2^-e for the byte above: exponent field 127 - e = 254 - byte, always normal.
__device__ __forceinline__ float inv_scale(uint32_t sb) { return __uint_as_float((254u - sb) << 23); }

// Eight fp32 values -> eight E2M1 codes in one word, element 0 in the lowest
// nibble.  cvt...e2m1x2 puts its first source in the high nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float a0, float a1, float a2, float a3, float a4, float a5,
                                               float a6, float a7)
{
    uint32_t r;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(r)
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
    return r;
}

// max(|a|, |b|, |c|) in one instruction (three-input max, sm_100).
__device__ __forceinline__ float max3_abs(float a, float b, float c)
{
    float r;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// max(|a|, |b|, |c|), NaN if any input is NaN (three-input max, sm_100).
__device__ __forceinline__ float max3_abs_nan(float a, float b, float c)
{
    float r;
    asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <bool NAN_>
__device__ __forceinline__ float max3_mag(float a, float b, float c)
{
    return NAN_ ? max3_abs_nan(a, b, c) : max3_abs(a, b, c);
}

// max |v(i)| over i < 32 as a tree of three-input maxes (depth 4), not a
// chain of 16 dependent ones: the block amax is on every quantizer's
// critical path, and inline-asm maxes are never reassociated by the
// compiler.  NAN_ selects the NaN-propagating form.
template <bool NAN_, class V>
__device__ __forceinline__ float amax32(V v)
{
    float m[11];
#pragma unroll
    for (int k = 0; k < 10; ++k) m[k] = max3_mag<NAN_>(v(3 * k), v(3 * k + 1), v(3 * k + 2));
    m[10] = max3_mag<NAN_>(v(30), v(31), 0.0f);
    const float n0 = max3_mag<NAN_>(m[0], m[1], m[2]);
    const float n1 = max3_mag<NAN_>(m[3], m[4], m[5]);
    const float n2 = max3_mag<NAN_>(m[6], m[7], m[8]);
    const float n3 = max3_mag<NAN_>(m[9], m[10], 0.0f);
    return max3_mag<NAN_>(max3_mag<NAN_>(n0, n1, n2), n3, 0.0f);
}

// The MXFP4 block quantizer on 32 fp32 values: amax, E8M0 byte, scaling by
// the exact power of two 2^-e, E2M1 rounding, packing.  A block with a value
// that is not finite gets the E8M0 NaN byte 0xFF and zero codes.
__device__ __forceinline__ void mx_quantize_block(const float (&v)[32], uint4 &codes, uint32_t &sbyte)
{
    const float amax = amax32<true>([&](int i) { return v[i]; });
    if (!(amax <= 3.40282347e38f)) {
        codes = make_uint4(0u, 0u, 0u, 0u);
        sbyte = 0xFFu;
        return;
    }
    const uint32_t sb = e8m0_byte(amax);
    const float s = inv_scale(sb);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
        w[q] = cvt_e2m1x8(v[8 * q] * s, v[8 * q + 1] * s, v[8 * q + 2] * s, v[8 * q + 3] * s,
                          v[8 * q + 4] * s, v[8 * q + 5] * s, v[8 * q + 6] * s, v[8 * q + 7] * s);
    codes = make_uint4(w[0], w[1], w[2], w[3]);
    sbyte = sb;
}

__device__ __forceinline__ void load_block(const uint4 *__restrict__ act, int64_t g, uint4 (&raw)[4])
{
    const uint4 *p = act + g * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) raw[q] = __ldg(p + q);
}

// ---------------------------------------------------------------------------
// kernels.  Grid: T threads (T = nb * R for the column-pinned kernels), each
// thread walks the flattened block index g = t, t + T, t + 2T, ... < nblocks.
// With T a multiple of nb the column j = g % nb is the same on every step, so
// a thread loads its column's factors (or multipliers) once.
// ---------------------------------------------------------------------------
enum class KqOut { kCodes, kF32 };

// Every kernel of the library begins with griddepcontrol.wait, and every
// launch allows programmatic stream serialization (launch() below): a kernel
// may then be scheduled while its predecessor on the stream finishes, but it
// touches no memory before that predecessor has completed and its writes are
// visible.  Launched without the attribute, the wait returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <KqOut OUT>
__global__ void __launch_bounds__(kThreads)
kq_butterfly_kernel(const uint4 *__restrict__ act, const float4 *__restrict__ factors, int shared,
                    uint4 *__restrict__ codes, uint8_t *__restrict__ scales, float4 *__restrict__ y_out,
                    int64_t nblocks, int nb, int64_t T)
{
    pdl_wait();
    const int64_t t = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    if (t >= T || t >= nblocks) return;
    const int j = int(t % nb);
    float f[20];
    const float4 *fp = factors + (shared ? 0 : int64_t(j) * 5);
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const float4 q = __ldg(fp + k);
        f[4 * k] = q.x;
        f[4 * k + 1] = q.y;
        f[4 * k + 2] = q.z;
        f[4 * k + 3] = q.w;
    }
    for (int64_t g = t; g < nblocks; g += T) {
        uint4 raw[4];
        load_block(act, g, raw);
        float v[32];
        unpack32(raw, v);
        kron_apply(v, f);
        if constexpr (OUT == KqOut::kCodes) {
            uint4 c;
            uint32_t sb;
            mx_quantize_block(v, c, sb);
            codes[g] = c;
            scales[g] = uint8_t(sb);
        } else {
            float4 *yo = y_out + g * 8;
#pragma unroll
            for (int q = 0; q < 8; ++q) yo[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    }
}

// Fold: w' = w K^-1 for a row vector w, i.e. w'^T = (K^-1)^T w^T, which is
// the Kronecker product of the 2x2 matrices (G_k^-1)^T = [[g11, -g10],
// [-g01, g00]] / det(G_k) applied as butterflies.  With INVERSE, the
// matrices are G_k^-1 = [[g11, -g01], [-g10, g00]] / det(G_k) instead, i.e.
// x = K^-1 y per block (the inverse transform).  fp32 in, fp32 out.
template <bool INVERSE>
__global__ void __launch_bounds__(kThreads)
fold_kernel(const float4 *__restrict__ W, const float4 *__restrict__ factors, int shared,
            float4 *__restrict__ W_out, int64_t nblocks, int nb, int64_t T)
{
    pdl_wait();
    const int64_t t = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    if (t >= T || t >= nblocks) return;
    const int j = int(t % nb);
    float f[20];
    const float4 *fp = factors + (shared ? 0 : int64_t(j) * 5);
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const float4 q = __ldg(fp + k);
        const float det = fmaf(q.x, q.w, -q.y * q.z);
        const float r = 1.0f / det;
        f[4 * k] = q.w * r;
        f[4 * k + 1] = (INVERSE ? -q.y : -q.z) * r;
        f[4 * k + 2] = (INVERSE ? -q.z : -q.y) * r;
        f[4 * k + 3] = q.x * r;
    }
    for (int64_t g = t; g < nblocks; g += T) {
        float v[32];
        const float4 *wp = W + g * 8;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 a = __ldg(wp + q);
            v[4 * q] = a.x;
            v[4 * q + 1] = a.y;
            v[4 * q + 2] = a.z;
            v[4 * q + 3] = a.w;
        }
        kron_apply(v, f);
        float4 *wo = W_out + g * 8;
#pragma unroll
        for (int q = 0; q < 8; ++q) wo[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
}

// ---------------------------------------------------------------------------
// Packed-pair kernels.  A block's 32 values sit in 16 register pairs
// p[i] = (x_i, x_{i+16}), so that every operation that treats the 32 values
// alike, or pairs index i with i ^ 2^b for b < 4, runs as one packed f32x2
// instruction on two values (__fmul2_rn / __ffma2_rn, sm_100).  Each thread
// prefetches the next block of its grid-stride walk before working on the
// current one, so two 64-byte loads per thread are in flight.
// ---------------------------------------------------------------------------

// p[i] = (x_i, x_{i+16}) from the 64 bytes of a block (raw[0..1] hold
// elements 0..15, raw[2..3] elements 16..31).
__device__ __forceinline__ void unpack_pairs(const uint4 (&raw)[4], float2 (&p)[16])
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t lo[4] = {raw[h].x, raw[h].y, raw[h].z, raw[h].w};
        const uint32_t hi[4] = {raw[h + 2].x, raw[h + 2].y, raw[h + 2].z, raw[h + 2].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            p[8 * h + 2 * w] = make_float2(bf16_lo(lo[w]), bf16_lo(hi[w]));
            p[8 * h + 2 * w + 1] = make_float2(bf16_hi(lo[w]), bf16_hi(hi[w]));
        }
    }
}

// The rest of the MXFP4 block quantizer on the pair layout once the amax is
// known: E8M0 byte from its exponent field, exact scaling by 2^-e, E2M1
// round-to-nearest-even with saturation, packing.
__device__ __forceinline__ void mx_finish_pairs(float2 (&p)[16], float amax, uint4 &codes, uint32_t &sbyte)
{
    const uint32_t sb = e8m0_byte(amax);
    const float s = inv_scale(sb);
    const float2 ss = make_float2(s, s);
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i] = __fmul2_rn(p[i], ss);
    codes.x = cvt_e2m1x8(p[0].x, p[1].x, p[2].x, p[3].x, p[4].x, p[5].x, p[6].x, p[7].x);
    codes.y = cvt_e2m1x8(p[8].x, p[9].x, p[10].x, p[11].x, p[12].x, p[13].x, p[14].x, p[15].x);
    codes.z = cvt_e2m1x8(p[0].y, p[1].y, p[2].y, p[3].y, p[4].y, p[5].y, p[6].y, p[7].y);
    codes.w = cvt_e2m1x8(p[8].y, p[9].y, p[10].y, p[11].y, p[12].y, p[13].y, p[14].y, p[15].y);
    sbyte = sb;
}

// MXFP4 block quantizer on the pair layout (same arithmetic as
// mx_quantize_block: amax, E8M0 byte from its exponent field, exact scaling
// by 2^-e, E2M1 round-to-nearest-even with saturation, packing).
__device__ __forceinline__ void mx_quantize_pairs(float2 (&p)[16], uint4 &codes, uint32_t &sbyte)
{
    const float amax = amax32<false>([&](int i) { return (i & 1) ? p[i >> 1].y : p[i >> 1].x; });
    mx_finish_pairs(p, amax, codes, sbyte);
}

// Block amax on the pair layout, NaN if any value is NaN.
__device__ __forceinline__ float pair_amax_nan(const float2 (&p)[16])
{
    return amax32<true>([&](int i) { return (i & 1) ? p[i >> 1].y : p[i >> 1].x; });
}

// Stage on in-block index bit b < 4 (pair-index distance S = 2^b) in unit-
// diagonal form: lo' = lo + b*hi, hi' = c*lo + hi (packed, both halves).
template <int S>
__device__ __forceinline__ void unit_stage2(float2 (&p)[16], float2 B, float2 C)
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (i & S) continue;
        const float2 lo = p[i], hi = p[i + S];
        p[i] = __ffma2_rn(B, hi, lo);
        p[i + S] = __ffma2_rn(C, lo, hi);
    }
}

// Stage on bit b < 4 in the direct form lo' = f00 lo + f01 hi, hi' = f10 lo + f11 hi.
template <int S>
__device__ __forceinline__ void direct_stage2(float2 (&p)[16], float2 F00, float2 F01, float2 F10, float2 F11)
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (i & S) continue;
        const float2 lo = p[i], hi = p[i + S];
        p[i] = __ffma2_rn(F01, hi, __fmul2_rn(F00, lo));
        p[i + S] = __ffma2_rn(F11, hi, __fmul2_rn(F10, lo));
    }
}

__device__ __forceinline__ float2 bcast(float v) { return make_float2(v, v); }

__device__ __forceinline__ float2 plus_zero2() { return make_float2(0.0f, 0.0f); }

// Unit-diagonal split of one factor; false if the factor is outside the range
// where the split is used (see the kernel comment).
__device__ __forceinline__ bool unit_split(const float4 g, float &d0, float &d1, float &b, float &c)
{
    d0 = g.x;
    d1 = g.w;
    b = __fdividef(g.y, g.x);
    c = __fdividef(g.z, g.w);
    const float a0 = fabsf(d0), a1 = fabsf(d1);
    return a0 >= 0x1p-16f && a0 <= 0x1p16f && a1 >= 0x1p-16f && a1 <= 0x1p16f && fabsf(b) <= 16.0f &&
           fabsf(c) <= 16.0f;
}

__device__ __forceinline__ void load_block_nc(const uint4 *__restrict__ act, int64_t g, uint4 (&raw)[4])
{
    const uint4 *p = act + g * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) raw[q] = __ldg(p + q);
}

// Column state of the KroQuant transform in unit-diagonal form (see the
// variant-2 kernel below for the derivation): the 32 values of D as 16 pairs
// (D_i, D_{i+16}) matching the register pairs of the data, and the
// off-diagonal coefficients of the five unit factors (scalars, used as
// broadcast operands of the packed instructions).
struct KqFast {
    float2 DP[16];            // (D_i, D_{i+16})
    float B[4], C[4];         // stages on bits 0..3 (G5, G4, G3, G2)
    float b4, c4;             // stage on bit 4 (G1)
};

__device__ __forceinline__ bool kq_fast_setup(const float4 (&g)[5], KqFast &st)
{
    float d0[5], d1[5], bb[5], cc[5];
    bool fast = true;
#pragma unroll
    for (int k = 0; k < 5; ++k) fast &= unit_split(g[k], d0[k], d1[k], bb[k], cc[k]);
    // D_i = prod_k (bit (4-k) of i ? g11_k : g00_k); factor k = 0 (G1) acts on bit 4.
    float dd[32];
    dd[0] = 1.0f;
#pragma unroll
    for (int bit = 0; bit < 5; ++bit) {
        const int k = 4 - bit;
#pragma unroll
        for (int i = 0; i < (1 << bit); ++i) {
            dd[i + (1 << bit)] = dd[i] * d1[k];
            dd[i] = dd[i] * d0[k];
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) st.DP[i] = make_float2(dd[i], dd[i + 16]);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        st.B[b] = bb[4 - b];
        st.C[b] = cc[4 - b];
    }
    st.b4 = bb[0];
    st.c4 = cc[0];
    return fast;
}

__device__ __forceinline__ void kq_fast_apply(float2 (&p)[16], const KqFast &st)
{
    unit_stage2<1>(p, bcast(st.B[0]), bcast(st.C[0]));
    unit_stage2<2>(p, bcast(st.B[1]), bcast(st.C[1]));
    unit_stage2<4>(p, bcast(st.B[2]), bcast(st.C[2]));
    unit_stage2<8>(p, bcast(st.B[3]), bcast(st.C[3]));
    // stage on bit 4, then D applied as D*z + (+0): the same value as D*z,
    // except that an exact zero comes out as +0 whatever the signs of D and z
    // (as a sum of products that cancels exactly does in round-to-nearest).
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float lo = p[i].x, hi = p[i].y;
        p[i] = __ffma2_rn(make_float2(fmaf(st.b4, hi, lo), fmaf(st.c4, lo, hi)), st.DP[i], plus_zero2());
    }
}

// The direct form, y_lo = g00 lo + g01 hi, y_hi = g10 lo + g11 hi per stage.
__device__ __forceinline__ void kq_direct_apply(float2 (&p)[16], const float4 (&g)[5])
{
    direct_stage2<1>(p, bcast(g[4].x), bcast(g[4].y), bcast(g[4].z), bcast(g[4].w));
    direct_stage2<2>(p, bcast(g[3].x), bcast(g[3].y), bcast(g[3].z), bcast(g[3].w));
    direct_stage2<4>(p, bcast(g[2].x), bcast(g[2].y), bcast(g[2].z), bcast(g[2].w));
    direct_stage2<8>(p, bcast(g[1].x), bcast(g[1].y), bcast(g[1].z), bcast(g[1].w));
    // last stage, with the same +0 canonicalisation of exact zeros
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float lo = p[i].x, hi = p[i].y;
        p[i] = __fadd2_rn(make_float2(fmaf(g[0].y, hi, g[0].x * lo), fmaf(g[0].w, hi, g[0].z * lo)),
                          plus_zero2());
    }
}

// Output of one transformed block: its MXFP4 codes and scale from the block
// amax (NaN-propagating; a non-finite block gets 0xFF and zero codes), or the
// fp32 values themselves.
template <KqOut OUT>
__device__ __forceinline__ void kq_emit(float2 (&p)[16], float amax, int64_t gi, uint4 *__restrict__ codes,
                                        uint8_t *__restrict__ scales, float4 *__restrict__ y_out)
{
    if constexpr (OUT == KqOut::kCodes) {
        uint4 c;
        uint32_t sb;
        if (amax <= 3.40282347e38f) {
            mx_finish_pairs(p, amax, c, sb);
        } else {
            c = make_uint4(0u, 0u, 0u, 0u);
            sb = 0xFFu;
        }
        codes[gi] = c;
        scales[gi] = uint8_t(sb);
    } else {
        float4 *yo = y_out + gi * 8;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            yo[q] = make_float4(p[4 * q].x, p[4 * q + 1].x, p[4 * q + 2].x, p[4 * q + 3].x);
            yo[q + 4] = make_float4(p[4 * q].y, p[4 * q + 1].y, p[4 * q + 2].y, p[4 * q + 3].y);
        }
    }
}

// Scale-factor layout of the block-scaled tensor-core MMA (PTX ISA, tcgen05
// block scaling, the scale-factor operand): the scales of 128 rows x 4
// consecutive blocks form one 512-byte unit, 32 lanes x 16 bytes, lane l
// holding rows l, l+32, l+64, l+96 at bytes 4*((r / 32) % 4), each as its 4
// blocks in order; units are ordered row-group major (the ceil(nb/4) units of
// 128 rows are consecutive).  For odd nb the byte of block column nb is
// written as 0x00 (2^-127): the MMA's last K=64 step reads it beside the real
// column nb-1, against zero codes, and it must be finite.
struct SfPos {
    int64_t row;     // current row (advances by rstep per step of the thread)
    int64_t rstep;
    int64_t ka512;   // 512 * ceil(nb / 4): bytes per 128-row group
    int64_t col;     // column part of the offset: 512 * (j / 4) + j % 4
    bool pad;        // this thread writes the odd-nb pad byte
};

__device__ __forceinline__ SfPos sf_pos(int64_t t, int64_t T, int nb)
{
    SfPos s;
    const int j = int(t % nb);
    s.row = t / nb;
    s.rstep = T / nb;
    s.ka512 = int64_t((nb + 3) >> 2) * 512;
    s.col = int64_t(j >> 2) * 512 + (j & 3);
    s.pad = (nb & 1) && j == nb - 1;
    return s;
}

__device__ __forceinline__ int64_t sf_offset(const SfPos &s)
{
    return (s.row >> 7) * s.ka512 + (s.row & 31) * 16 + ((s.row >> 5) & 3) * 4 + s.col;
}

// Codes as kq_emit; the scale byte at its scale-factor-layout offset.
__device__ __forceinline__ void kq_emit_sf(float2 (&p)[16], float amax, int64_t gi, uint4 *__restrict__ codes,
                                           uint8_t *__restrict__ sf, SfPos &sp)
{
    uint4 c;
    uint32_t sb;
    if (amax <= 3.40282347e38f) {
        mx_finish_pairs(p, amax, c, sb);
    } else {
        c = make_uint4(0u, 0u, 0u, 0u);
        sb = 0xFFu;
    }
    codes[gi] = c;
    const int64_t off = sf_offset(sp);
    sf[off] = uint8_t(sb);
    if (sp.pad) sf[off + 1] = 0;
    sp.row += sp.rstep;
}

__device__ __forceinline__ void load_factors(const float4 *__restrict__ factors, int shared, int j, float4 (&g)[5])
{
    const float4 *fp = factors + (shared ? 0 : int64_t(j) * 5);
#pragma unroll
    for (int k = 0; k < 5; ++k) g[k] = __ldg(fp + k);
}

// The factors from the LU form of KroQuant section 3.2, Eq. (6): G = L U with
// U = [[a, b], [0, -1/a]] and L = [[1, 0], [c, 1]], i.e.
// G = [[a, b], [c a, c b - 1/a]]: 15 scalars per block (a, b, c per factor)
// expanded once per thread (the paper's on-the-fly "K2" reconstruction).
__device__ __forceinline__ void load_lu(const float *__restrict__ lu, int shared, int j, float4 (&g)[5])
{
    const float *pp = lu + (shared ? 0 : int64_t(j) * 15);
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const float a = __ldg(pp + 3 * k), b = __ldg(pp + 3 * k + 1), c = __ldg(pp + 3 * k + 2);
        g[k] = make_float4(a, b, c * a, fmaf(c, b, -(1.0f / a)));
    }
}

// The unit-diagonal form's intermediates (U x) can exceed the block's final
// values by up to 17^5 (|b|, |c| <= 16 per stage), so a finite block can
// overflow there while the direct form and the oracle stay finite.  The
// unit-diagonal loops only note that a block's amax came out non-finite
// (the NaN-propagating amax) and emit it as a non-finite block; after its
// loop, a thread that noted one walks its blocks start, start + stride, ...
// again and rewrites every block whose unit-diagonal amax is not finite with
// the direct form's result (0xFF and zero codes where that is not finite
// either).  Only inputs within 2^21 of the top of the fp32 range get here,
// and the loops keep no registers for it.
template <KqOut OUT, bool LU, bool SF>
__device__ __noinline__ void kq_redo_overflow(const uint4 *__restrict__ act, const float *__restrict__ params,
                                              int shared, int64_t start, int64_t stride, int64_t nblocks, int nb,
                                              uint4 *__restrict__ codes, uint8_t *__restrict__ scales,
                                              float4 *__restrict__ y_out)
{
    const int j = int(start % nb);
    float4 g[5];
    if constexpr (LU)
        load_lu(params, shared, j, g);
    else
        load_factors(reinterpret_cast<const float4 *>(params), shared, j, g);
    KqFast st;
    kq_fast_setup(g, st);
    SfPos sp{};
    if constexpr (SF) sp = sf_pos(start, stride, nb);
    for (int64_t gi = start; gi < nblocks; gi += stride) {
        uint4 raw[4];
        load_block_nc(act, gi, raw);
        float2 p[16];
        unpack_pairs(raw, p);
        kq_fast_apply(p, st);
        if (pair_amax_nan(p) <= 3.40282347e38f) {
            if constexpr (SF) sp.row += sp.rstep;
            continue;
        }
        unpack_pairs(raw, p);
        kq_direct_apply(p, g);
        if constexpr (SF)
            kq_emit_sf(p, pair_amax_nan(p), gi, codes, scales, sp);
        else
            kq_emit<OUT>(p, pair_amax_nan(p), gi, codes, scales, y_out);
    }
}

// KroQuant quantizer, packed butterfly (variant 2).
//
// Each 2x2 factor is split as G = [[g00, g01], [g10, g11]]
// = diag(g00, g11) [[1, b], [c, 1]] with b = g01/g00, c = g10/g11; by the
// mixed-product property K = G1 (x) ... (x) G5 = D U, with D the diagonal
// (x)_k diag(g00_k, g11_k) and U = (x)_k [[1, b_k], [c_k, 1]].  A unit-diagonal
// stage costs one FFMA per element and D one multiply, so the transform and
// scaling take 7 FP32 lane operations per element against 11 for the direct
// form.  The rounding differs from the direct form by a few fp32 ulps of
// (|K||x|)_i, the same order as the direct form's own rounding.
// A thread whose column has a factor with |g00| or |g11| outside
// [2^-16, 2^16] or |b| or |c| above 16 (where U's intermediate values could
// grow by more than 17^5) runs the direct form instead.
// With SF the scales go to the scale-factor layout (requires T a multiple of
// nb, as the pinned geometry gives).
template <KqOut OUT, bool LU = false, bool SF = false>
__global__ void __launch_bounds__(kThreads, 2)
kq_packed_kernel(const uint4 *__restrict__ act, const float *__restrict__ params, int shared,
                 uint4 *__restrict__ codes, uint8_t *__restrict__ scales, float4 *__restrict__ y_out,
                 int64_t nblocks, int nb, int64_t T)
{
    pdl_wait();
    const int64_t t = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    if (t >= T || t >= nblocks) return;
    SfPos sp{};
    if constexpr (SF) sp = sf_pos(t, T, nb);
    // the first block's load goes out before the column set-up, so the two
    // latencies (activation from HBM, factors from L2) overlap
    int64_t gi = t;
    uint4 raw[4];
    load_block_nc(act, gi, raw);
    const int j = int(t % nb);
    float4 g[5];
    if constexpr (LU)
        load_lu(params, shared, j, g);
    else
        load_factors(reinterpret_cast<const float4 *>(params), shared, j, g);
    KqFast st;
    const bool fast = kq_fast_setup(g, st);
    bool overflow = false;
    if (fast) {
        for (;;) {
            const int64_t gn = gi + T;
            uint4 nxt[4];
            if (gn < nblocks) load_block_nc(act, gn, nxt);
            float2 p[16];
            unpack_pairs(raw, p);
            kq_fast_apply(p, st);
            const float amax = pair_amax_nan(p);
            overflow |= !(amax <= 3.40282347e38f);
            if constexpr (SF)
                kq_emit_sf(p, amax, gi, codes, scales, sp);
            else
                kq_emit<OUT>(p, amax, gi, codes, scales, y_out);
            if (gn >= nblocks) break;
#pragma unroll
            for (int q = 0; q < 4; ++q) raw[q] = nxt[q];
            gi = gn;
        }
    } else {
        for (;;) {
            const int64_t gn = gi + T;
            uint4 nxt[4];
            if (gn < nblocks) load_block_nc(act, gn, nxt);
            float2 p[16];
            unpack_pairs(raw, p);
            kq_direct_apply(p, g);
            if constexpr (SF)
                kq_emit_sf(p, pair_amax_nan(p), gi, codes, scales, sp);
            else
                kq_emit<OUT>(p, pair_amax_nan(p), gi, codes, scales, y_out);
            if (gn >= nblocks) break;
#pragma unroll
            for (int q = 0; q < 4; ++q) raw[q] = nxt[q];
            gi = gn;
        }
    }
    if (overflow) kq_redo_overflow<OUT, LU, SF>(act, params, shared, t, T, nblocks, nb, codes, scales, y_out);
}

// Fixed-Hadamard baseline (the transform the pages compare the on-the-fly
// kernel against): y = H_H x / sqrt(H) on every H consecutive channels, H =
// 2^(5 + xstages) in [32, 1024], H | d, with H_H the Sylvester matrix
// (H2 (x) ... (x) H2), then the MXFP4 quantizer on each 32-block.  A thread
// holds one 32-block: the five stages on its in-block index bits are
// in-register (lo + hi, lo - hi); an H-block spans H/32 consecutive lanes of a
// warp, and each further stage exchanges all 32 values with the partner lane
// lane ^ 2^s by shuffles.  Warps walk the flattened block array together (the
// grid stride is a multiple of 32, so the lanes of an H-block stay aligned).
template <int S>
__device__ __forceinline__ void hadamard_stage2(float2 (&p)[16])
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (i & S) continue;
        const float2 lo = p[i], hi = p[i + S];
        p[i] = __fadd2_rn(lo, hi);
        p[i + S] = __ffma2_rn(hi, make_float2(-1.0f, -1.0f), lo);
    }
}

__global__ void __launch_bounds__(kThreads)
fwht_kernel(const uint4 *__restrict__ act, uint4 *__restrict__ codes, uint8_t *__restrict__ scales, int64_t nblocks,
            int64_t T, int xstages, float inv_sqrt_h)
{
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t t0 = int64_t(blockIdx.x) * kThreads + (threadIdx.x & ~31);   // the warp's first thread
    for (int64_t g0 = t0; g0 < nblocks; g0 += T) {                            // warp-uniform walk
        const int64_t gi = g0 + lane;
        const bool valid = gi < nblocks;       // whole H-blocks are valid or not (H | d)
        uint4 raw[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                        make_uint4(0, 0, 0, 0)};
        if (valid) load_block_nc(act, gi, raw);
        float2 p[16];
        unpack_pairs(raw, p);
        hadamard_stage2<1>(p);
        hadamard_stage2<2>(p);
        hadamard_stage2<4>(p);
        hadamard_stage2<8>(p);
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = make_float2(p[i].x + p[i].y, p[i].x - p[i].y);
#pragma unroll
        for (int s = 0; s < 5; ++s) {
            if (s >= xstages) break;
            const int m = 1 << s;
            const float sg = (lane & m) ? -1.0f : 1.0f;   // partner holds the other half of the pair
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float ox = __shfl_xor_sync(0xffffffffu, p[i].x, m);
                const float oy = __shfl_xor_sync(0xffffffffu, p[i].y, m);
                p[i] = make_float2(fmaf(sg, p[i].x, ox), fmaf(sg, p[i].y, oy));
            }
        }
        const float2 nrm = make_float2(inv_sqrt_h, inv_sqrt_h);
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = __fmul2_rn(p[i], nrm);
        if (valid) {
            uint4 c;
            uint32_t sb;
            mx_quantize_pairs(p, c, sb);
            codes[gi] = c;
            scales[gi] = uint8_t(sb);
        }
    }
}

// SmoothQuant quantizer on the pair layout: y = fp32(x * m) per channel (one
// correctly rounded packed multiply), then the MXFP4 block quantizer.
__global__ void __launch_bounds__(kThreads)
sq_packed_kernel(const uint4 *__restrict__ act, const float4 *__restrict__ mult, uint4 *__restrict__ codes,
                 uint8_t *__restrict__ scales, int64_t nblocks, int nb, int64_t T)
{
    pdl_wait();
    const int64_t t = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    if (t >= T || t >= nblocks) return;
    const int j = int(t % nb);
    float m[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 a = __ldg(mult + int64_t(j) * 8 + q);
        m[4 * q] = a.x;
        m[4 * q + 1] = a.y;
        m[4 * q + 2] = a.z;
        m[4 * q + 3] = a.w;
    }
    float2 MP[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) MP[i] = make_float2(m[i], m[i + 16]);
    int64_t gi = t;
    uint4 raw[4];
    load_block_nc(act, gi, raw);
    for (;;) {
        const int64_t gn = gi + T;
        uint4 nxt[4];
        if (gn < nblocks) load_block_nc(act, gn, nxt);
        float2 p[16];
        unpack_pairs(raw, p);
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = __fmul2_rn(p[i], MP[i]);
        uint4 c;
        uint32_t sb;
        mx_quantize_pairs(p, c, sb);
        codes[gi] = c;
        scales[gi] = uint8_t(sb);
        if (gn >= nblocks) break;
#pragma unroll
        for (int q = 0; q < 4; ++q) raw[q] = nxt[q];
        gi = gn;
    }
}

// Plain MXFP4 quantizer on the pair layout.
__global__ void __launch_bounds__(kThreads)
mx_packed_kernel(const uint4 *__restrict__ act, uint4 *__restrict__ codes, uint8_t *__restrict__ scales,
                 int64_t nblocks, int64_t T)
{
    pdl_wait();
    const int64_t t = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    if (t >= nblocks) return;
    int64_t gi = t;
    uint4 raw[4];
    load_block_nc(act, gi, raw);
    for (;;) {
        const int64_t gn = gi + T;
        uint4 nxt[4];
        if (gn < nblocks) load_block_nc(act, gn, nxt);
        float2 p[16];
        unpack_pairs(raw, p);
        uint4 c;
        uint32_t sb;
        mx_quantize_pairs(p, c, sb);
        codes[gi] = c;
        scales[gi] = uint8_t(sb);
        if (gn >= nblocks) break;
#pragma unroll
        for (int q = 0; q < 4; ++q) raw[q] = nxt[q];
        gi = gn;
    }
}

// ---------------------------------------------------------------------------
// TMA-staged kernels.  The activation, viewed as a [nblocks][32] bf16 matrix
// (one 64-byte row per block), streams through a ring of kStages
// shared-memory stages of kStageRows rows each: one producer thread issues a
// 2-D tensor copy (cp.async.bulk.tensor) per stage and mbarriers hand stages
// between it and the consumer warps.  So the bytes in flight per SM no longer
// depend on registers (2 CTAs x 4 stages x 16 KB), unlike a register
// prefetch.  The copies use the 64-byte swizzle: the 16-byte chunk q of row r
// lands at chunk q ^ ((r >> 1) & 3), which makes the consumers' 16-byte
// shared loads (8 lanes per phase reading 8 consecutive rows) conflict-free.
// Every wait is bounded by a clock budget; a wait that gives up records it
// in g_wait_timeouts, and the kernel drains its copies in flight (again
// bounded) before it returns, so a fault elsewhere cannot hang the GPU here.
// ---------------------------------------------------------------------------
constexpr int kStageRows = 256;                        // blocks per stage: one per consumer thread
constexpr int kStageBytes = kStageRows * 64;           // 16 KB
constexpr int kStages = 4;
constexpr int kConsumers = 256;
constexpr int kStagedThreads = kConsumers + 32;        // + one producer warp
constexpr size_t kStagedSmem = size_t(kStages) * kStageBytes + 1024 + 2 * kStages * sizeof(uint64_t);

__device__ int g_wait_timeouts;

// Operand of kq_selftest_bounded_wait: its tensor map covers kSelftestBlocks
// rows of 64 bytes, and the same array stands in for the codes (16 B per
// block) and scales (1 B per block) outputs, so it spans the whole map even
// though that launch issues no copies and writes nothing.
constexpr int64_t kSelftestBlocks = int64_t(kStageRows) * (kStages + 1);
__device__ __align__(256) uint8_t g_selftest_dummy[kSelftestBlocks * 64];
static_assert(sizeof(g_selftest_dummy) >= kSelftestBlocks * 64, "selftest map and outputs stay inside the array");

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done)
                 : "r"(smem_addr(bar)), "r"(parity)
                 : "memory");
    return done != 0;
}

// Wait for the phase with the given parity to complete; false if `budget`
// clock cycles pass first (the caller then records the timeout and unwinds).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long budget)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > budget) return false;
    return true;
}

__device__ __forceinline__ void tma_load_rows(void *dst, const CUtensorMap *map, int32_t row, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row), "r"(smem_addr(bar))
        : "memory");
}

struct StagedRing {
    uint8_t *stage;
    uint64_t *full;
    uint64_t *empty;
};

// Carve the ring out of dynamic shared memory (stages aligned to 1 KB for the
// swizzle) and initialise the barriers; every thread of the CTA calls this.
__device__ __forceinline__ StagedRing staged_setup()
{
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    StagedRing r;
    r.stage = base;
    r.full = reinterpret_cast<uint64_t *>(base + size_t(kStages) * kStageBytes);
    r.empty = r.full + kStages;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&r.full[s], 1);
            mbar_init(&r.empty[s], kConsumers / 32);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    return r;
}

// Producer (one thread): fill stage k % kStages with chunk c = blockIdx.x +
// k * gridDim.x, after the consumers have released the stage's previous use.
// issue_copies == 0 issues nothing (used only to test the bounded waits).
__device__ void staged_produce(const StagedRing &r, const CUtensorMap *map, int64_t nchunks, long long budget,
                               int issue_copies)
{
    int k = 0;
    int filled = 0;                          // number of fills issued
    for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++k) {
        const int s = k % kStages;
        if (k >= kStages && !mbar_wait(&r.empty[s], ((k / kStages) - 1) & 1, budget)) {
            atomicAdd(&g_wait_timeouts, 1);
            break;
        }
        if (!issue_copies) continue;
        mbar_expect_tx(&r.full[s], kStageBytes);
        tma_load_rows(r.stage + size_t(s) * kStageBytes, map, int32_t(c * kStageRows), &r.full[s]);
        filled = k + 1;
    }
    // Drain: every issued copy has landed before this thread (and so the CTA)
    // can exit.  On the normal path the consumers have waited on all of them.
    for (int kk = (filled > kStages ? filled - kStages : 0); kk < filled; ++kk) {
        if (!mbar_wait(&r.full[kk % kStages], (kk / kStages) & 1, budget)) {
            atomicAdd(&g_wait_timeouts, 1);
            break;
        }
    }
}

// Consumer loop: thread tid owns row tid of every stage, i.e. block
// g = c * kStageRows + tid.  f(raw, g) runs for the rows below nblocks.
// Returns false after a timeout (recorded).
template <class F>
__device__ __forceinline__ bool staged_consume(const StagedRing &r, int64_t nchunks, int64_t nblocks, long long budget,
                                               F &&f)
{
    const int tid = threadIdx.x;
    const int sw = (tid >> 1) & 3;
    int k = 0;
    for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++k) {
        const int s = k % kStages;
        if (!mbar_wait(&r.full[s], (k / kStages) & 1, budget)) {
            atomicAdd(&g_wait_timeouts, 1);
            return false;
        }
        const uint8_t *row = r.stage + size_t(s) * kStageBytes + size_t(tid) * 64;
        uint4 raw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) raw[q] = *reinterpret_cast<const uint4 *>(row + 16 * (q ^ sw));
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(&r.empty[s]);
        const int64_t g = c * kStageRows + tid;
        if (g < nblocks) f(raw, g);
    }
    return true;
}

// KroQuant quantizer, TMA-staged (variant 3): the arithmetic of variant 2
// (kq_fast_apply / kq_direct_apply) on blocks read from the staged ring.
// The grid is a multiple of nb / gcd(nb, kStageRows), so gridDim.x *
// kStageRows is a multiple of nb and a thread's column j never changes.
__global__ void __launch_bounds__(kStagedThreads, 2)
kq_staged_kernel(const __grid_constant__ CUtensorMap act_map, const uint4 *__restrict__ act,
                 const float4 *__restrict__ factors, int shared,
                 uint4 *__restrict__ codes, uint8_t *__restrict__ scales, int64_t nblocks, int nb,
                 long long budget, int issue_copies)
{
    pdl_wait();
    const StagedRing r = staged_setup();
    const int64_t nchunks = (nblocks + kStageRows - 1) / kStageRows;
    if (threadIdx.x >= kConsumers) {
        if (threadIdx.x == kConsumers) staged_produce(r, &act_map, nchunks, budget, issue_copies);
        return;
    }
    const int j = int((int64_t(blockIdx.x) * kStageRows + threadIdx.x) % nb);
    float4 g[5];
    load_factors(factors, shared, j, g);
    KqFast st;
    if (kq_fast_setup(g, st)) {
        bool overflow = false;
        staged_consume(r, nchunks, nblocks, budget, [&](const uint4 (&raw)[4], int64_t gi) {
            float2 p[16];
            unpack_pairs(raw, p);
            kq_fast_apply(p, st);
            const float amax = pair_amax_nan(p);
            overflow |= !(amax <= 3.40282347e38f);
            kq_emit<KqOut::kCodes>(p, amax, gi, codes, scales, nullptr);
        });
        if (overflow)
            kq_redo_overflow<KqOut::kCodes, false, false>(
                act, reinterpret_cast<const float *>(factors), shared, int64_t(blockIdx.x) * kStageRows + threadIdx.x,
                int64_t(gridDim.x) * kStageRows, nblocks, nb, codes, scales, nullptr);
    } else {
        staged_consume(r, nchunks, nblocks, budget, [&](const uint4 (&raw)[4], int64_t gi) {
            float2 p[16];
            unpack_pairs(raw, p);
            kq_direct_apply(p, g);
            kq_emit<KqOut::kCodes>(p, pair_amax_nan(p), gi, codes, scales, nullptr);
        });
    }
}

// SmoothQuant quantizer, TMA-staged.
__global__ void __launch_bounds__(kStagedThreads, 2)
sq_staged_kernel(const __grid_constant__ CUtensorMap act_map, const float4 *__restrict__ mult,
                 uint4 *__restrict__ codes, uint8_t *__restrict__ scales, int64_t nblocks, int nb, long long budget,
                 int issue_copies)
{
    pdl_wait();
    const StagedRing r = staged_setup();
    const int64_t nchunks = (nblocks + kStageRows - 1) / kStageRows;
    if (threadIdx.x >= kConsumers) {
        if (threadIdx.x == kConsumers) staged_produce(r, &act_map, nchunks, budget, issue_copies);
        return;
    }
    const int j = int((int64_t(blockIdx.x) * kStageRows + threadIdx.x) % nb);
    float m[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 a = __ldg(mult + int64_t(j) * 8 + q);
        m[4 * q] = a.x;
        m[4 * q + 1] = a.y;
        m[4 * q + 2] = a.z;
        m[4 * q + 3] = a.w;
    }
    float2 MP[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) MP[i] = make_float2(m[i], m[i + 16]);
    staged_consume(r, nchunks, nblocks, budget, [&](const uint4 (&raw)[4], int64_t gi) {
        float2 p[16];
        unpack_pairs(raw, p);
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = __fmul2_rn(p[i], MP[i]);
        uint4 c;
        uint32_t sb;
        mx_quantize_pairs(p, c, sb);
        codes[gi] = c;
        scales[gi] = uint8_t(sb);
    });
}

// Plain MXFP4 quantizer, TMA-staged.
__global__ void __launch_bounds__(kStagedThreads, 2)
mx_staged_kernel(const __grid_constant__ CUtensorMap act_map, uint4 *__restrict__ codes,
                 uint8_t *__restrict__ scales, int64_t nblocks, long long budget, int issue_copies)
{
    pdl_wait();
    const StagedRing r = staged_setup();
    const int64_t nchunks = (nblocks + kStageRows - 1) / kStageRows;
    if (threadIdx.x >= kConsumers) {
        if (threadIdx.x == kConsumers) staged_produce(r, &act_map, nchunks, budget, issue_copies);
        return;
    }
    staged_consume(r, nchunks, nblocks, budget, [&](const uint4 (&raw)[4], int64_t gi) {
        float2 p[16];
        unpack_pairs(raw, p);
        uint4 c;
        uint32_t sb;
        mx_quantize_pairs(p, c, sb);
        codes[gi] = c;
        scales[gi] = uint8_t(sb);
    });
}

// MXFP4 decode (the consumer side of the quantizers): value = E2M1(code) *
// 2^(byte - 127), exact in fp32 (two significant bits times a power of two;
// byte 0 gives the subnormal 2^-127, byte 0xFF is NaN).  The codes go
// through the hardware E2M1 -> f16x2 conversion (exact: every E2M1 value is
// an f16 value).
__device__ __forceinline__ float2 e2m1x2_to_f32x2(uint32_t byte)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 q;\n\tcvt.u8.u32 q, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, q;\n\t}" : "=r"(h2) : "r"(byte));
    const __half2 h = *reinterpret_cast<const __half2 *>(&h2);
    return make_float2(__low2float(h), __high2float(h));
}

__device__ __forceinline__ float e8m0_value(uint32_t sb)
{
    if (sb == 0xFFu) return __uint_as_float(0x7fc00000u);
    return sb ? __uint_as_float(sb << 23) : __uint_as_float(0x00400000u);
}

__global__ void __launch_bounds__(kThreads)
mx_dequantize_kernel(const uint4 *__restrict__ codes, const uint8_t *__restrict__ scales, float4 *__restrict__ out,
                     int64_t nblocks)
{
    pdl_wait();
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    for (int64_t g = int64_t(blockIdx.x) * kThreads + threadIdx.x; g < nblocks; g += stride) {
        const uint4 c = __ldg(codes + g);
        const float s = e8m0_value(__ldg(scales + g));
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        float v[32];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const float2 e = e2m1x2_to_f32x2((w[q] >> (8 * b)) & 0xFFu);   // low nibble = even element
                v[8 * q + 2 * b] = e.x * s;
                v[8 * q + 2 * b + 1] = e.y * s;
            }
        float4 *o = out + g * 8;
#pragma unroll
        for (int q = 0; q < 8; ++q) o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
}

// Plain MXFP4 quantizer on fp32 input, for the folded weights W T^-1 of
// KroQuant section 3.2, Eq. (4) (fp32 after the fold): one 32-block per
// thread, the same block quantizer as the activation kernels; scales
// row-major [M][nb] or, with SF, in the scale-factor layout.
template <bool SF>
__global__ void __launch_bounds__(kThreads)
mx_f32_kernel(const float4 *__restrict__ x, uint4 *__restrict__ codes, uint8_t *__restrict__ scales,
              int64_t nblocks, int nb)
{
    pdl_wait();
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    for (int64_t g = int64_t(blockIdx.x) * kThreads + threadIdx.x; g < nblocks; g += stride) {
        float v[32];
        const float4 *src = x + g * 8;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 f = __ldg(src + q);
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
        uint4 c;
        uint32_t sb;
        mx_quantize_block(v, c, sb);
        codes[g] = c;
        if constexpr (SF) {
            SfPos sp = sf_pos(g, g + 1, nb);   // row g / nb, column g % nb (rstep unused)
            const int64_t off = sf_offset(sp);
            scales[off] = uint8_t(sb);
            if (sp.pad) scales[off + 1] = 0;
        } else {
            scales[g] = uint8_t(sb);
        }
    }
}

// Row-major scales [M][nb] -> the scale-factor layout (one byte per thread),
// with the odd-nb pad byte; lets every quantizer feed the W4A4 product.
__global__ void __launch_bounds__(kThreads)
sf_relayout_kernel(const uint8_t *__restrict__ scales, uint8_t *__restrict__ sf, int64_t n, int nb)
{
    pdl_wait();
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    for (int64_t g = int64_t(blockIdx.x) * kThreads + threadIdx.x; g < n; g += stride) {
        SfPos sp = sf_pos(g, g + 1, nb);
        const int64_t off = sf_offset(sp);
        sf[off] = __ldg(scales + g);
        if (sp.pad) sf[off + 1] = 0;
    }
}

// 16-byte global -> shared copy through L2 only (cp.async, no register staging).
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *g)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}


// The quantizer fused with the normalisation that produces its input (KroQuant
// abstract: normalisation layers force the transform online).  For every token
// row h of a bf16 activation: LayerNorm without affine (mean, biased
// variance, eps inside the square root), AdaLN modulation
// x_mod = LN(h) (1 + gamma_b) + beta_b with per-sample vectors (rows grouped by
// sample, rows_per consecutive rows each), then the KroQuant transform and
// MXFP4 -- x_mod never leaves registers.
//
// One warp per row.  Pass 1 streams the row from HBM; each lane folds the
// blocks it reads into a running (count, mean, sum of squared deviations)
// with the parallel-variance combination of Chan, Golub and LeVeque, and five
// shuffle steps merge the lanes.  Pass 2 reads the row again (from L2: a row is
// at most 32 KB and a wave of warps touches a few MB) and quantizes every
// block with its column's coefficients, which the CTA computes once into a
// shared-memory table: per column the 16 D pairs, the 10 off-diagonal
// coefficients, a flag for the unit-diagonal form and the 20 raw factors (the
// direct-form fallback), kNormSlot floats, an odd number of 16-byte units so
// lanes reading consecutive columns hit distinct bank groups.
constexpr int kNormSlot = 68;   // 32 DP + 12 (coefficients, flag, pad) + 20 raw + 4 pad = 272 B

struct Welford {
    float n, mean, m2;
};

__device__ __forceinline__ Welford welford_merge(Welford a, Welford b)
{
    const float n = a.n + b.n;
    if (n == 0.0f) return a;
    const float delta = b.mean - a.mean;
    const float fb = b.n / n;
    Welford r;
    r.n = n;
    r.mean = fmaf(delta, fb, a.mean);
    r.m2 = a.m2 + b.m2 + delta * delta * a.n * fb;
    return r;
}

// Codes and scale of block (r, j); with SF the scale byte goes to the
// scale-factor layout (see SfPos), with the odd-nb pad byte.
template <bool SF>
__device__ __forceinline__ void norm_emit(float2 (&p)[16], int64_t r, int j, int nb, uint4 *__restrict__ codes,
                                          uint8_t *__restrict__ scales)
{
    if constexpr (SF) {
        uint4 c;
        uint32_t sb;
        mx_quantize_pairs(p, c, sb);
        codes[r * nb + j] = c;
        const int64_t off = (r >> 7) * (int64_t((nb + 3) >> 2) * 512) + (r & 31) * 16 + ((r >> 5) & 3) * 4 +
                            int64_t(j >> 2) * 512 + (j & 3);
        scales[off] = uint8_t(sb);
        if ((nb & 1) && j == nb - 1) scales[off + 1] = 0;
    } else {
        kq_emit<KqOut::kCodes>(p, pair_amax_nan(p), r * nb + j, codes, scales, nullptr);
    }
}

template <bool SF>
__global__ void __launch_bounds__(kThreads)
norm_kq_kernel(const uint4 *__restrict__ h, const float *__restrict__ gamma, const float *__restrict__ beta,
               int64_t rows_per, float eps, const float *__restrict__ factors, int shared, uint4 *__restrict__ codes,
               uint8_t *__restrict__ scales, int64_t M, int nb)
{
    pdl_wait();
    extern __shared__ __align__(16) float tab[];   // [nb][kNormSlot]
    // coefficient table (every column of the row, computed once per CTA)
    for (int j = threadIdx.x; j < nb; j += blockDim.x) {
        float4 g[5];
        load_factors(reinterpret_cast<const float4 *>(factors), shared, j, g);
        KqFast st;
        const bool fast = kq_fast_setup(g, st);
        float *e = tab + j * kNormSlot;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            e[2 * i] = st.DP[i].x;
            e[2 * i + 1] = st.DP[i].y;
        }
        float4 *q = reinterpret_cast<float4 *>(e + 32);
        q[0] = make_float4(st.B[0], st.C[0], st.B[1], st.C[1]);
        q[1] = make_float4(st.B[2], st.C[2], st.B[3], st.C[3]);
        q[2] = make_float4(st.b4, st.c4, fast ? 1.0f : 0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < 5; ++k) q[3 + k] = g[k];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int d = nb * kBlk;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t r = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32; r < M; r += warps) {
        const uint4 *hrow = h + r * nb * 4;
        // ---- pass 1: row statistics
        Welford w = {0.0f, 0.0f, 0.0f};
        for (int j = lane; j < nb; j += 32) {
            uint4 raw[4];
            load_block_nc(hrow, j, raw);
            float2 p[16];
            unpack_pairs(raw, p);
            float2 s2 = p[0];
#pragma unroll
            for (int i = 1; i < 16; ++i) s2 = __fadd2_rn(s2, p[i]);
            const float bmean = (s2.x + s2.y) * (1.0f / 32.0f);
            const float2 nm = make_float2(-bmean, -bmean);
            float2 q2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float2 t = __fadd2_rn(p[i], nm);
                q2 = __ffma2_rn(t, t, q2);
            }
            w = welford_merge(w, Welford{32.0f, bmean, q2.x + q2.y});
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            Welford o;
            o.n = __shfl_xor_sync(0xffffffffu, w.n, off);
            o.mean = __shfl_xor_sync(0xffffffffu, w.mean, off);
            o.m2 = __shfl_xor_sync(0xffffffffu, w.m2, off);
            w = welford_merge(w, o);
        }
        const float mu = w.mean;
        const float inv = 1.0f / sqrtf(w.m2 / float(d) + eps);
        // ---- pass 2: normalise, modulate, transform, quantize
        const int64_t b = r / rows_per;
        const float2 nmu = make_float2(-mu, -mu), iv = make_float2(inv, inv);
        for (int j = lane; j < nb; j += 32) {
            uint4 raw[4];
            load_block_nc(hrow, j, raw);
            float2 p[16];
            unpack_pairs(raw, p);
            const float4 *gp = reinterpret_cast<const float4 *>(gamma + b * d + j * kBlk);
            const float4 *bp = reinterpret_cast<const float4 *>(beta + b * d + j * kBlk);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 ga = __ldg(gp + q4), gb = __ldg(gp + q4 + 4);
                const float4 ba = __ldg(bp + q4), bb = __ldg(bp + q4 + 4);
                const float g_lo[4] = {ga.x, ga.y, ga.z, ga.w}, g_hi[4] = {gb.x, gb.y, gb.z, gb.w};
                const float b_lo[4] = {ba.x, ba.y, ba.z, ba.w}, b_hi[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 4 * q4 + e;
                    const float2 t = __fmul2_rn(__fadd2_rn(p[i], nmu), iv);
                    p[i] = __ffma2_rn(t, make_float2(1.0f + g_lo[e], 1.0f + g_hi[e]), make_float2(b_lo[e], b_hi[e]));
                }
            }
            const float4 *eq = reinterpret_cast<const float4 *>(tab + j * kNormSlot);
            const float4 c4q = eq[10];
            if (c4q.z != 0.0f) {
                const float4 c01 = eq[8], c23 = eq[9];
                unit_stage2<1>(p, bcast(c01.x), bcast(c01.y));
                unit_stage2<2>(p, bcast(c01.z), bcast(c01.w));
                unit_stage2<4>(p, bcast(c23.x), bcast(c23.y));
                unit_stage2<8>(p, bcast(c23.z), bcast(c23.w));
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 dd = eq[q];   // (D_2q, D_2q+16, D_2q+1, D_2q+17)
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int i = 2 * q + h2;
                        const float lo = p[i].x, hi = p[i].y;
                        const float2 dp = h2 ? make_float2(dd.z, dd.w) : make_float2(dd.x, dd.y);
                        p[i] = __ffma2_rn(make_float2(fmaf(c4q.x, hi, lo), fmaf(c4q.y, lo, hi)), dp, plus_zero2());
                    }
                }
            } else {
                float4 g[5];
#pragma unroll
                for (int k = 0; k < 5; ++k) g[k] = eq[11 + k];
                kq_direct_apply(p, g);
            }
            norm_emit<SF>(p, r, j, nb, codes, scales);
        }
    }
}

// Single-pass form of the fused normalisation + quantizer, used wherever its
// shared memory fits (the kernel above is the general fallback).  Each CTA
// owns a contiguous range of rows of one sample; its shared-memory table holds,
// per column, the unit-stage coefficients of K = U' D and that sample's
// D (1 + gamma) and D beta, the transform's diagonal folded into the
// modulation (kNormRowSlot float4, an odd number of 16-byte units; a column in
// the direct form, which is rare, keeps 1 + gamma and beta and reloads its raw
// factors).  Each warp
// streams whole rows into a ring of nbuf row buffers with cp.async (every
// instruction of a warp copies 512 contiguous bytes; the 16-byte piece p of
// block b lands at b * 64 + 16 (p ^ ((b >> 1) & 3)), so the per-lane block
// reads of the second sweep are free of bank conflicts), the next row in
// flight while the current one is processed: the row is read from HBM once.
// From shared memory a warp takes the sums of x and x^2 in one sweep (a
// second sweep over (x - mu)^2 only where the mean is large against the root
// mean square), then normalises, modulates, transforms and quantizes every
// block.
constexpr int kNormRowSlot = 19;   // 2 B/C + 1 (b4, c4, flag) + 8 D (1 + gamma) + 8 D beta

template <bool SF>
__global__ void __launch_bounds__(512, 1)
norm_kq_rows_kernel(const uint4 *__restrict__ h, const float *__restrict__ gamma, const float *__restrict__ beta,
                    int64_t rows_per, float eps, const float *__restrict__ factors, int shared,
                    uint4 *__restrict__ codes, uint8_t *__restrict__ scales, int nb, int cps, int nbuf)
{
    pdl_wait();
    extern __shared__ float4 smf[];
    float4 *tab = smf;                                                        // [nb][kNormRowSlot]
    uint4 *rowbuf = reinterpret_cast<uint4 *>(smf + size_t(nb) * kNormRowSlot);   // [warps][nbuf][nb * 4]
    const int warps = int(blockDim.x) / 32, wid = int(threadIdx.x) / 32, lane = int(threadIdx.x) & 31;
    const int64_t smp = blockIdx.x / cps;
    const int part = int(blockIdx.x % cps);
    const int64_t r0 = smp * rows_per + rows_per * part / cps;
    const int64_t r1 = smp * rows_per + rows_per * (part + 1) / cps;
    const int d = nb * kBlk;
    // The transform in the form K = U' D (as the long-row kernel): each factor
    // G = [[1, g01 / g11], [g10 / g00, 1]] diag(g00, g11), so D acts first and
    // folds into the modulation, whose table entry holds D (1 + gamma) and
    // D beta + 0 (+0 for a zero product: no intermediate is ever -0, and an
    // exactly cancelling sum comes out +0); the five unit stages of U' follow,
    // with no D multiply per element.  A column the split does not admit keeps
    // 1 + gamma and beta and runs the direct form.  Entry layout: [0], [1] the
    // (b, c) of the stages on bits 0-3, [2] (b, c) of bit 4 and the flag,
    // [3 + q] D (1 + gamma) and [11 + q] D beta for elements 4q .. 4q + 3.
    for (int j = threadIdx.x; j < nb; j += blockDim.x) {
        float4 g[5];
        load_factors(reinterpret_cast<const float4 *>(factors), shared, j, g);
        float d0[5], d1[5], bk[5], ck[5];
        bool fast = true;
#pragma unroll
        for (int k = 0; k < 5; ++k) {
            d0[k] = g[k].x;
            d1[k] = g[k].w;
            bk[k] = __fdividef(g[k].y, g[k].w);
            ck[k] = __fdividef(g[k].z, g[k].x);
            const float a0 = fabsf(d0[k]), a1 = fabsf(d1[k]);
            fast &= a0 >= 0x1p-16f && a0 <= 0x1p16f && a1 >= 0x1p-16f && a1 <= 0x1p16f && fabsf(bk[k]) <= 16.0f &&
                    fabsf(ck[k]) <= 16.0f;
        }
        float dd[32];
        dd[0] = 1.0f;
#pragma unroll
        for (int bit = 0; bit < 5; ++bit) {
            const int k = 4 - bit;
#pragma unroll
            for (int i = 0; i < (1 << bit); ++i) {
                dd[i + (1 << bit)] = dd[i] * d1[k];
                dd[i] = dd[i] * d0[k];
            }
        }
        float4 *e = tab + size_t(j) * kNormRowSlot;
        // factor k (G_{k+1}) acts on in-block index bit 4 - k
        e[0] = make_float4(bk[4], ck[4], bk[3], ck[3]);
        e[1] = make_float4(bk[2], ck[2], bk[1], ck[1]);
        e[2] = make_float4(bk[0], ck[0], fast ? 1.0f : 0.0f, 0.0f);
        const float4 *gp = reinterpret_cast<const float4 *>(gamma + smp * d + int64_t(j) * kBlk);
        const float4 *bp = reinterpret_cast<const float4 *>(beta + smp * d + int64_t(j) * kBlk);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 ga = __ldg(gp + q);
            const float4 ba = __ldg(bp + q);
            float4 gg = make_float4(1.0f + ga.x, 1.0f + ga.y, 1.0f + ga.z, 1.0f + ga.w);
            float4 bb = ba;
            if (fast) {
                gg = make_float4(dd[4 * q] * gg.x, dd[4 * q + 1] * gg.y, dd[4 * q + 2] * gg.z, dd[4 * q + 3] * gg.w);
                bb = make_float4(fmaf(dd[4 * q], bb.x, 0.0f), fmaf(dd[4 * q + 1], bb.y, 0.0f),
                                 fmaf(dd[4 * q + 2], bb.z, 0.0f), fmaf(dd[4 * q + 3], bb.w, 0.0f));
            }
            e[3 + q] = gg;
            e[11 + q] = bb;
        }
    }
    __syncthreads();

    const int npieces = nb * 4;                                   // 16-byte pieces per row
    uint4 *wbuf = rowbuf + size_t(wid) * nbuf * npieces;
    const uint32_t wbase = static_cast<uint32_t>(__cvta_generic_to_shared(wbuf));
    const int64_t nrows = (r1 - r0 > wid) ? (r1 - r0 - wid + warps - 1) / warps : 0;   // this warp's rows
    // Piece c = lane + 32 k is piece (lane & 3) of block (lane >> 2) + 8 k, whose
    // swizzle term ((block >> 1) & 3) = (lane >> 3) & 3 does not depend on k: a
    // lane's pieces sit at a fixed offset plus 512 k bytes.
    const int lslot = (lane & ~3) + ((lane & 3) ^ ((lane >> 3) & 3));
    const int nk = (npieces - lane + 31) / 32;                    // this lane's pieces per row
    auto issue = [&](int64_t r, int buf) {
        const uint4 *src = h + r * npieces + lane;
        uint32_t dst = wbase + uint32_t((buf * npieces + lslot) * 16);
        for (int k = 0; k < nk; ++k, src += 32, dst += 512) cp_async16(dst, src);
    };
    if (nrows > 0) issue(r0 + wid, 0);
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t r = r0 + wid + i * warps;
        const int buf = nbuf == 2 ? int(i & 1) : 0;
        if (nbuf == 2) {
            if (i + 1 < nrows) issue(r + warps, buf ^ 1);
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            if (i > 0) {
                issue(r, 0);
                asm volatile("cp.async.commit_group;" ::: "memory");
            }
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();
        const uint4 *rb = wbuf + size_t(buf) * npieces;
        // ---- statistics.  One sweep gives the sums of x and x^2; where the mean
        // is small against the root mean square (mu^2 <= 2^-6 E[x^2]) the
        // variance E[x^2] - mu^2 loses at most ~2 ulp to cancellation and is
        // used directly, otherwise a second sweep sums (x - mu)^2 (the
        // two-pass variance).  The choice is warp-uniform (reduced values).
        const uint4 *lp = rb + lslot;                             // this lane's pieces, 32 apart
        float2 s2 = make_float2(0.0f, 0.0f), q2 = make_float2(0.0f, 0.0f);
        for (int k = 0; k < nk; ++k) {
            const uint4 w = lp[32 * k];
            float2 t;
            t = make_float2(bf16_lo(w.x), bf16_hi(w.x));
            s2 = __fadd2_rn(s2, t);
            q2 = __ffma2_rn(t, t, q2);
            t = make_float2(bf16_lo(w.y), bf16_hi(w.y));
            s2 = __fadd2_rn(s2, t);
            q2 = __ffma2_rn(t, t, q2);
            t = make_float2(bf16_lo(w.z), bf16_hi(w.z));
            s2 = __fadd2_rn(s2, t);
            q2 = __ffma2_rn(t, t, q2);
            t = make_float2(bf16_lo(w.w), bf16_hi(w.w));
            s2 = __fadd2_rn(s2, t);
            q2 = __ffma2_rn(t, t, q2);
        }
        float sum = s2.x + s2.y, sq = q2.x + q2.y;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const float mu = sum / float(d);
        const float2 nmu = make_float2(-mu, -mu);
        const float ex2 = sq / float(d);
        float m2;
        if (mu * mu <= ex2 * (1.0f / 64.0f)) {
            m2 = fmaxf(ex2 - mu * mu, 0.0f) * float(d);
        } else {
            q2 = make_float2(0.0f, 0.0f);
            for (int k = 0; k < nk; ++k) {
                const uint4 w = lp[32 * k];
                float2 t;
                t = __fadd2_rn(make_float2(bf16_lo(w.x), bf16_hi(w.x)), nmu);
                q2 = __ffma2_rn(t, t, q2);
                t = __fadd2_rn(make_float2(bf16_lo(w.y), bf16_hi(w.y)), nmu);
                q2 = __ffma2_rn(t, t, q2);
                t = __fadd2_rn(make_float2(bf16_lo(w.z), bf16_hi(w.z)), nmu);
                q2 = __ffma2_rn(t, t, q2);
                t = __fadd2_rn(make_float2(bf16_lo(w.w), bf16_hi(w.w)), nmu);
                q2 = __ffma2_rn(t, t, q2);
            }
            m2 = q2.x + q2.y;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m2 += __shfl_xor_sync(0xffffffffu, m2, off);
        }
        // x / sigma - mu / sigma as one FMA (the product x / sigma is exact inside
        // it, so the result differs from (x - mu) / sigma by one rounding of
        // mu / sigma), as in the long-row kernel
        const float inv = __frsqrt_rn(fmaf(m2, 1.0f / float(d), eps));
        const float2 iv = make_float2(inv, inv);
        const float2 off = make_float2(-mu * inv, -mu * inv);
        // ---- normalise, modulate, transform, quantize
        for (int jb = lane; jb < nb; jb += 32) {
            uint4 raw[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) raw[q] = rb[jb * 4 + (q ^ ((jb >> 1) & 3))];
            float2 p[16];
            unpack_pairs(raw, p);
            const float4 *eq = tab + size_t(jb) * kNormRowSlot;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 ga = eq[3 + q4], gb = eq[7 + q4], ba = eq[11 + q4], bb = eq[15 + q4];
                const float g_lo[4] = {ga.x, ga.y, ga.z, ga.w}, g_hi[4] = {gb.x, gb.y, gb.z, gb.w};
                const float b_lo[4] = {ba.x, ba.y, ba.z, ba.w}, b_hi[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i2 = 4 * q4 + e;
                    const float2 t = __ffma2_rn(p[i2], iv, off);
                    p[i2] = __ffma2_rn(t, make_float2(g_lo[e], g_hi[e]), make_float2(b_lo[e], b_hi[e]));
                }
            }
            const float4 c4q = eq[2];
            if (c4q.z != 0.0f) {
                const float4 c01 = eq[0], c23 = eq[1];
                unit_stage2<1>(p, bcast(c01.x), bcast(c01.y));
                unit_stage2<2>(p, bcast(c01.z), bcast(c01.w));
                unit_stage2<4>(p, bcast(c23.x), bcast(c23.y));
                unit_stage2<8>(p, bcast(c23.z), bcast(c23.w));
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float lo = p[i].x, hi = p[i].y;
                    p[i] = make_float2(fmaf(c4q.x, hi, lo), fmaf(c4q.y, lo, hi));
                }
            } else {   // rare: the raw factors, from L1
                float4 g[5];
                load_factors(reinterpret_cast<const float4 *>(factors), shared, jb, g);
                kq_direct_apply(p, g);
            }
            norm_emit<SF>(p, r, jb, nb, codes, scales);
        }
        __syncwarp();   // every lane is done with the buffer before it is refilled
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

#include "kq_mma.cuh"
#include "kq_ring.cuh"
#include "mxf4_gemm.cuh"

// Third form of the fused normalisation + quantizer, for long rows (where the
// per-column table and whole-row buffers of the single-pass kernel do not
// fit, or fit for too few warps): a CTA takes two rows of its sample at a
// time, thread t owning block column t (blockDim = nb rounded up to a warp),
// and holds the two rows' blocks as register pairs p[i] = (row a x_i, row b
// x_i), as the two-row ring quantizer does: every stage of the transform and
// every step of the normalisation is one packed f32x2 instruction for both
// rows, and the two rows are independent chains.  A thread's column never
// changes, so its transform coefficients sit in registers, and its sample's
// 1 + gamma and beta in a shared-memory table laid out [q][t] (float4 q of
// thread t), conflict-free for a warp.  Each thread streams its own 64-byte
// block of every row through a DEPTH-row cp.async ring in shared memory (a
// CTA's copies of a row are contiguous; the 16-byte piece p of thread t lands
// at t * 64 + 16 (p ^ ((t >> 1) & 3)), so the reads back are conflict-free),
// DEPTH - 2 rows ahead of the pair it transforms: each row is read from HBM
// once, without a register prefetch.  The row statistics are a CTA reduction:
// per warp a shuffle reduction of both rows' sums, per CTA the warps' partial
// sums in a shared array double-buffered by step parity, so one barrier per
// two rows suffices (a second one only on the two-pass branch).  Per element:
// x / sigma - mu / sigma (one FMA), times D (1 + gamma) plus D beta (one FMA:
// the transform's diagonal folded into the modulation), the five unit stages
// of K = U' D, MXFP4: seven FMA-pipe operations from x to y, where the
// other two kernels take nine.
template <bool SF>
__device__ __forceinline__ void norm_store(uint4 c, uint32_t sb, int64_t r, int j, int nb, uint4 *__restrict__ codes,
                                           uint8_t *__restrict__ scales)
{
    codes[r * nb + j] = c;
    if constexpr (SF) {
        const int64_t off = (r >> 7) * (int64_t((nb + 3) >> 2) * 512) + (r & 31) * 16 + ((r >> 5) & 3) * 4 +
                            int64_t(j >> 2) * 512 + (j & 3);
        scales[off] = uint8_t(sb);
        if ((nb & 1) && j == nb - 1) scales[off + 1] = 0;
    } else {
        scales[r * nb + j] = uint8_t(sb);
    }
}

template <bool SF, int DEPTH, int kMaxThreads>
__global__ void __launch_bounds__(kMaxThreads, 1)
norm_kq_cols_kernel(const uint4 *__restrict__ h, const float *__restrict__ gamma, const float *__restrict__ beta,
                    int64_t rows_per, float eps, const float *__restrict__ factors, int shared,
                    uint4 *__restrict__ codes, uint8_t *__restrict__ scales, int nb, int cps)
{
    pdl_wait();
    static_assert(DEPTH % 2 == 0 && DEPTH >= 2, "the ring holds whole pairs of rows");
    extern __shared__ float4 smc[];
    const int nt = int(blockDim.x);                                        // threads = nb rounded up to 32
    const int t = int(threadIdx.x), wid = t >> 5, lane = t & 31, nw = nt >> 5;
    float4 *gtab = smc;                                                    // [8][nt] (1 + gamma)
    float4 *btab = smc + 8 * nt;                                           // [8][nt] beta
    uint4 *ring = reinterpret_cast<uint4 *>(smc + 16 * nt);                // [DEPTH][nt * 4]
    float4 *red = reinterpret_cast<float4 *>(ring + DEPTH * nt * 4);       // [2][nw] (sums, squares) of a, b
    float2 *red2 = reinterpret_cast<float2 *>(red + 2 * nw);               // [2][nw] (x - mu)^2 sums of a, b
    const int64_t smp = blockIdx.x / cps;
    const int part = int(blockIdx.x % cps);
    const int64_t r0 = smp * rows_per + rows_per * part / cps;
    const int64_t r1 = smp * rows_per + rows_per * (part + 1) / cps;
    const int d = nb * kBlk;
    const float inv_d = 1.0f / float(d);
    const bool active = t < nb;
    const int j = active ? t : 0;

    // this thread's copies of row r into ring slot `slot` (16-byte pieces, swizzled)
    const uint32_t rbase = static_cast<uint32_t>(__cvta_generic_to_shared(ring)) + uint32_t(t) * 64;
    const int sw = (t >> 1) & 3;
    auto issue = [&](int64_t r, int slot) {
        if (active && r < r1) {
            const uint4 *src = h + (r * nb + t) * 4;
            const uint32_t dst = rbase + uint32_t(slot) * uint32_t(nt) * 64;
#pragma unroll
            for (int q = 0; q < 4; ++q) cp_async16(dst + 16 * (q ^ sw), src + q);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // the first rows go out before the set-up
#pragma unroll
    for (int k = 0; k < DEPTH; ++k) issue(r0 + k, k);

    // The transform in the form K = U' D: each factor G = [[1, g01 / g11], [g10 /
    // g00, 1]] diag(g00, g11), so the diagonal D (the same as in K = D U) acts
    // first and folds into the modulation: x'' = t (D (1 + gamma)) + D beta,
    // then the five unit stages of U' -- no D multiply per element.  The table
    // holds D (1 + gamma) and D beta + 0 (+0 for a zero product, so no
    // intermediate is ever -0 and an exactly cancelling sum comes out +0).
    // A column whose factors the split does not admit keeps 1 + gamma and beta
    // in the table and runs the direct form.
    float B[5], C[5];
    bool fast = true;
    const float *gsm = gamma + smp * d + int64_t(j) * kBlk;
    const float *bsm = beta + smp * d + int64_t(j) * kBlk;
    {
        float4 g[5];
        load_factors(reinterpret_cast<const float4 *>(factors), shared, j, g);
        float d0[5], d1[5];
#pragma unroll
        for (int k = 0; k < 5; ++k) {
            d0[k] = g[k].x;
            d1[k] = g[k].w;
            const float bk = __fdividef(g[k].y, g[k].w), ck = __fdividef(g[k].z, g[k].x);
            const float a0 = fabsf(d0[k]), a1 = fabsf(d1[k]);
            fast &= a0 >= 0x1p-16f && a0 <= 0x1p16f && a1 >= 0x1p-16f && a1 <= 0x1p16f && fabsf(bk) <= 16.0f &&
                    fabsf(ck) <= 16.0f;
            B[4 - k] = bk;           // factor k (G_{k+1}) acts on in-block index bit 4 - k
            C[4 - k] = ck;
        }
        float dd[32];
        dd[0] = 1.0f;
#pragma unroll
        for (int bit = 0; bit < 5; ++bit) {
            const int k = 4 - bit;
#pragma unroll
            for (int i = 0; i < (1 << bit); ++i) {
                dd[i + (1 << bit)] = dd[i] * d1[k];
                dd[i] = dd[i] * d0[k];
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 ga = active ? __ldg(reinterpret_cast<const float4 *>(gsm) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 ba = active ? __ldg(reinterpret_cast<const float4 *>(bsm) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            float4 gg = make_float4(1.0f + ga.x, 1.0f + ga.y, 1.0f + ga.z, 1.0f + ga.w);
            float4 bb = ba;
            if (fast) {
                gg = make_float4(dd[4 * q] * gg.x, dd[4 * q + 1] * gg.y, dd[4 * q + 2] * gg.z, dd[4 * q + 3] * gg.w);
                bb = make_float4(fmaf(dd[4 * q], bb.x, 0.0f), fmaf(dd[4 * q + 1], bb.y, 0.0f),
                                 fmaf(dd[4 * q + 2], bb.z, 0.0f), fmaf(dd[4 * q + 3], bb.w, 0.0f));
            }
            gtab[q * nt + t] = gg;
            btab[q * nt + t] = bb;
        }
    }

    int step = 0;
    for (int64_t ra = r0; ra < r1; ra += 2, ++step) {
        const int64_t rb = ra + 1;
        const bool two = rb < r1;
        const int sa = int((ra - r0) % DEPTH), sb = sa + 1;
        // rows ra and rb have landed (DEPTH - 2 younger groups may be in flight)
        asm volatile("cp.async.wait_group %0;" ::"n"(DEPTH - 2) : "memory");
        uint4 xa[4], xb[4];
        const uint4 *pa = ring + size_t(sa) * nt * 4 + size_t(t) * 4;
        const uint4 *pb = ring + size_t(sb) * nt * 4 + size_t(t) * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            xa[q] = active ? pa[q ^ sw] : make_uint4(0u, 0u, 0u, 0u);
            xb[q] = (active && two) ? pb[q ^ sw] : make_uint4(0u, 0u, 0u, 0u);
        }
        // the slots are read: refill them with the rows DEPTH ahead
        issue(ra + DEPTH, sa);
        issue(rb + DEPTH, sb);
        float2 p[32];
        ring::unpack_rows(xa, xb, p);
        // ---- statistics of both rows (one sweep of sums; the two-pass variance
        // where the mean is large against the root mean square, as the row kernel)
        // four partial sums each, so the additions are four short chains
        float2 sa4[4], qa4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            sa4[k] = p[k];
            qa4[k] = __fmul2_rn(p[k], p[k]);
        }
#pragma unroll
        for (int k = 4; k < 32; ++k) {
            sa4[k & 3] = __fadd2_rn(sa4[k & 3], p[k]);
            qa4[k & 3] = __ffma2_rn(p[k], p[k], qa4[k & 3]);
        }
        float2 s2 = __fadd2_rn(__fadd2_rn(sa4[0], sa4[1]), __fadd2_rn(sa4[2], sa4[3]));
        float2 q2 = __fadd2_rn(__fadd2_rn(qa4[0], qa4[1]), __fadd2_rn(qa4[2], qa4[3]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            s2.x += __shfl_xor_sync(0xffffffffu, s2.x, off);
            s2.y += __shfl_xor_sync(0xffffffffu, s2.y, off);
            q2.x += __shfl_xor_sync(0xffffffffu, q2.x, off);
            q2.y += __shfl_xor_sync(0xffffffffu, q2.y, off);
        }
        const int par = step & 1;
        if (lane == 0) red[par * nw + wid] = make_float4(s2.x, s2.y, q2.x, q2.y);
        __syncthreads();
        float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int w = 0; w < nw; ++w) {
            const float4 v = red[par * nw + w];
            tot.x += v.x;
            tot.y += v.y;
            tot.z += v.z;
            tot.w += v.w;
        }
        const float2 mu = make_float2(tot.x * inv_d, tot.y * inv_d);
        const float2 ex2 = make_float2(tot.z * inv_d, tot.w * inv_d);
        const float2 nmu = make_float2(-mu.x, -mu.y);
        float2 m2;
        // uniform over the CTA: the same totals everywhere
        if (mu.x * mu.x <= ex2.x * (1.0f / 64.0f) && mu.y * mu.y <= ex2.y * (1.0f / 64.0f)) {
            m2 = make_float2(fmaxf(ex2.x - mu.x * mu.x, 0.0f) * float(d), fmaxf(ex2.y - mu.y * mu.y, 0.0f) * float(d));
        } else {
            float2 c2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float2 tt = __fadd2_rn(p[k], nmu);
                c2 = __ffma2_rn(tt, tt, c2);
            }
            if (!active) c2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                c2.x += __shfl_xor_sync(0xffffffffu, c2.x, off);
                c2.y += __shfl_xor_sync(0xffffffffu, c2.y, off);
            }
            if (lane == 0) red2[par * nw + wid] = c2;
            __syncthreads();
            float2 two_pass = make_float2(0.f, 0.f);
            for (int w = 0; w < nw; ++w) {
                const float2 v = red2[par * nw + w];
                two_pass.x += v.x;
                two_pass.y += v.y;
            }
            // each row keeps the one-sweep value where its own mean allows it
            m2.x = mu.x * mu.x <= ex2.x * (1.0f / 64.0f) ? fmaxf(ex2.x - mu.x * mu.x, 0.0f) * float(d) : two_pass.x;
            m2.y = mu.y * mu.y <= ex2.y * (1.0f / 64.0f) ? fmaxf(ex2.y - mu.y * mu.y, 0.0f) * float(d) : two_pass.y;
        }
        if (!active) continue;
        const float2 iv = make_float2(__frsqrt_rn(fmaf(m2.x, inv_d, eps)), __frsqrt_rn(fmaf(m2.y, inv_d, eps)));
        // ---- normalise, modulate (both rows): x / sigma - mu / sigma as one
        // FMA (the product x / sigma is exact inside it, so the result differs
        // from (x - mu) / sigma by one rounding of mu / sigma), then times
        // 1 + gamma plus beta; transform, quantize
        const float2 off = make_float2(-mu.x * iv.x, -mu.y * iv.y);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 ga = gtab[q * nt + t], ba = btab[q * nt + t];
            const float gg[4] = {ga.x, ga.y, ga.z, ga.w}, bb[4] = {ba.x, ba.y, ba.z, ba.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 4 * q + e;
                const float2 tt = __ffma2_rn(p[i], iv, off);
                p[i] = __ffma2_rn(tt, make_float2(gg[e], gg[e]), make_float2(bb[e], bb[e]));
            }
        }
        if (fast) {
            ring::unit_stage<1>(p, B[0], C[0]);
            ring::unit_stage<2>(p, B[1], C[1]);
            ring::unit_stage<4>(p, B[2], C[2]);
            ring::unit_stage<8>(p, B[3], C[3]);
            ring::unit_stage<16>(p, B[4], C[4]);
        } else {   // rare: the raw factors, from L1
            float4 g[5];
            load_factors(reinterpret_cast<const float4 *>(factors), shared, j, g);
            ring::direct_apply(p, g);
        }
        float a0, a1;
        ring::amax_rows(p, a0, a1);
        uint4 c0, c1;
        uint32_t b0, b1;
        ring::finish_rows(p, a0, a1, c0, c1, b0, b1);
        if (!(a0 <= 3.40282347e38f)) {
            c0 = make_uint4(0u, 0u, 0u, 0u);
            b0 = 0xFFu;
        }
        if (!(a1 <= 3.40282347e38f)) {
            c1 = make_uint4(0u, 0u, 0u, 0u);
            b1 = 0xFFu;
        }
        norm_store<SF>(c0, b0, ra, t, nb, codes, scales);
        if (two) norm_store<SF>(c1, b1, rb, t, nb, codes, scales);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// ---------------------------------------------------------------------------
// launch geometry
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

int sm_count(int *out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev >= 0 && dev < kMaxDevices) {
        int c = g_sm_count[dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *out = c;
            return KQ_OK;
        }
    }
    int c = 0;
    e = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(c, std::memory_order_relaxed);
    *out = c;
    return KQ_OK;
}

// Threads T = nb * R with R rows per sweep chosen so that every thread runs
// the same number of steps, ceil(M / R), and T stays near the resident-thread
// target of the device.
struct Geometry {
    int64_t T;
    unsigned grid;
};

Geometry pinned_geometry(int64_t M, int64_t nb, int64_t target_threads)
{
    int64_t R = target_threads / nb;
    if (R < 1) R = 1;
    if (R > M) R = M;
    const int64_t steps = (M + R - 1) / R;
    R = (M + steps - 1) / steps;
    Geometry g;
    g.T = nb * R;
    g.grid = unsigned((g.T + kThreads - 1) / kThreads);
    return g;
}

// Resident threads of a kernel on the current device: SMs x resident CTAs
// per SM (occupancy query, cached per device and kernel).
enum KernelId {
    kKqDirect, kKqDirectF32, kKqPacked, kKqPackedF32, kSqPacked, kMxPacked, kFold,
    kKqStaged, kSqStaged, kMxStaged, kKqMma, kKqMmaF32, kKqLu, kFwht, kInverse, kDequant, kNormKq,
    kKqPackedSf, kMxF32, kMxF32Sf, kSfRelayout, kNormRows, kNormKqSf, kKqRing, kNumKernels
};
std::atomic<int> g_ctas_per_sm[kNumKernels][kMaxDevices];

int resident_threads(KernelId id, const void *fn, int64_t *out)
{
    int sms = 0;
    int rc = sm_count(&sms);
    if (rc != KQ_OK) return rc;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    int c = (dev >= 0 && dev < kMaxDevices) ? g_ctas_per_sm[id][dev].load(std::memory_order_relaxed) : 0;
    if (c <= 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c, fn, kThreads, 0);
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
        if (c < 1) c = 1;
        if (dev >= 0 && dev < kMaxDevices) g_ctas_per_sm[id][dev].store(c, std::memory_order_relaxed);
    }
    *out = int64_t(sms) * c * kThreads;
    return KQ_OK;
}

// Launch with programmatic stream serialization (see pdl_wait); a launch
// error is left for launch_check, as with the <<< >>> form.
template <typename... P, typename... A>
void launch(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, A &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

int launch_check(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
    return ok();
}

// Common argument checks; returns KQ_OK, an error status, or 1 for "no work".
int check_quant_args(const char *fn, const void *act, const void *params, bool need_params, const void *codes,
                     const void *scales, int64_t M, int64_t d)
{
    if (M < 0 || d <= 0 || d % kBlk != 0)
        return fail(KQ_ERR_SHAPE, "%s: need M >= 0 and d a positive multiple of 32 (M=%lld, d=%lld)", fn,
                    (long long)M, (long long)d);
    if (d / kBlk > INT32_MAX || (M > 0 && M > INT64_MAX / d))
        return fail(KQ_ERR_SHAPE, "%s: size too large (M=%lld, d=%lld)", fn, (long long)M, (long long)d);
    if (M == 0) return 1;
    if (!act || !codes || !scales || (need_params && !params))
        return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    if (!aligned(act, 16) || !aligned(codes, 16) || (need_params && !aligned(params, 16)))
        return fail(KQ_ERR_ALIGN, "%s: act, out_codes and factors/mult must be 16-byte aligned", fn);
    return KQ_OK;
}

// --- TMA-staged launches -----------------------------------------------------
// cuTensorMapEncodeTiled is looked up through the runtime, so the library
// needs no link-time dependency on the driver library.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::atomic<EncodeTiledFn> g_encode{nullptr};

int encode_fn(EncodeTiledFn *out)
{
    EncodeTiledFn f = g_encode.load(std::memory_order_acquire);
    if (!f) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled not available: %s", cudaGetErrorString(e));
        f = reinterpret_cast<EncodeTiledFn>(p);
        g_encode.store(f, std::memory_order_release);
    }
    *out = f;
    return KQ_OK;
}

// The activation as a [nblocks][32] bf16 matrix, boxes of kStageRows rows,
// 64-byte swizzle (the row is exactly one 64-byte swizzle span).
int encode_act_map(const void *act, int64_t nblocks, CUtensorMap *map, int box_rows = kStageRows)
{
    EncodeTiledFn enc;
    int rc = encode_fn(&enc);
    if (rc != KQ_OK) return rc;
    const cuuint64_t dims[2] = {32, cuuint64_t(nblocks)};
    const cuuint64_t strides[1] = {64};
    const cuuint32_t box[2] = {32, cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(act), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return KQ_OK;
}

std::atomic<int> g_smem_set[kNumKernels][kMaxDevices];
constexpr size_t kNormRowsSmemMax = size_t(227) * 1024;
std::atomic<int> g_norm_cfg[2][kMaxDevices][513];   // chosen single-pass norm configuration per row width

// Dynamic shared memory above 48 KB needs an opt-in per kernel and device.
int staged_prepare(KernelId id, const void *fn, int64_t *ctas_total)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices || !g_smem_set[id][dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kStagedSmem));
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        if (dev >= 0 && dev < kMaxDevices) g_smem_set[id][dev].store(1, std::memory_order_release);
    }
    int sms = 0;
    int rc = sm_count(&sms);
    if (rc != KQ_OK) return rc;
    int c = (dev >= 0 && dev < kMaxDevices) ? g_ctas_per_sm[id][dev].load(std::memory_order_relaxed) : 0;
    if (c <= 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c, fn, kStagedThreads, kStagedSmem);
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
        if (c < 1) c = 1;
        if (dev >= 0 && dev < kMaxDevices) g_ctas_per_sm[id][dev].store(c, std::memory_order_relaxed);
    }
    *ctas_total = int64_t(sms) * c;
    return KQ_OK;
}

int64_t gcd64(int64_t a, int64_t b)
{
    while (b) {
        const int64_t t = a % b;
        a = b;
        b = t;
    }
    return a;
}

// Grid of the staged kernels: a multiple of q = nb / gcd(nb, kStageRows), so
// that gridDim.x * kStageRows is a multiple of nb (fixed column per thread),
// as close to the resident-CTA count as that allows and no larger than the
// work needs.
unsigned staged_grid(int64_t nblocks, int64_t nb, int64_t resident)
{
    const int64_t q = nb / gcd64(nb, kStageRows);
    const int64_t nchunks = (nblocks + kStageRows - 1) / kStageRows;
    int64_t grid = (resident / q) * q;
    if (grid < q) grid = q;
    const int64_t need = ((nchunks + q - 1) / q) * q;
    if (grid > need) grid = need;
    return unsigned(grid);
}

// The activation as the [M][d] bf16 matrix, boxes of {64 columns x 128 rows}
// with the 128-byte swizzle (the A operand layout of the tcgen05 variant).
int encode_act_map_rows(const void *act, int64_t M, int64_t d, CUtensorMap *map)
{
    EncodeTiledFn enc;
    int rc = encode_fn(&enc);
    if (rc != KQ_OK) return rc;
    const cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(M)};
    const cuuint64_t strides[1] = {cuuint64_t(d) * 2};
    const cuuint32_t box[2] = {64, cuuint32_t(mma::kRows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(act), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return KQ_OK;
}

// The codes as the [M][d/2] uint8 matrix, boxes of {kNC*16 bytes x 32 rows}
// (one epilogue warp's rows of a tile of the tcgen05 variant), no swizzle.
int encode_codes_map(void *codes, int64_t M, int64_t d, CUtensorMap *map)
{
    EncodeTiledFn enc;
    int rc = encode_fn(&enc);
    if (rc != KQ_OK) return rc;
    const cuuint64_t dims[2] = {cuuint64_t(d / 2), cuuint64_t(M)};
    const cuuint64_t strides[1] = {cuuint64_t(d / 2)};
    const cuuint32_t box[2] = {cuuint32_t(mma::kNC * 16), cuuint32_t(mma::kStoreRows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return KQ_OK;
}

int mma_prepare(KernelId id, const void *fn)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices || !g_smem_set[id][dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(mma::kSmem));
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        if (dev >= 0 && dev < kMaxDevices) g_smem_set[id][dev].store(1, std::memory_order_release);
    }
    return KQ_OK;
}

int smem_prepare(KernelId id, const void *fn, size_t bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices || !g_smem_set[id][dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        if (dev >= 0 && dev < kMaxDevices) g_smem_set[id][dev].store(1, std::memory_order_release);
    }
    return KQ_OK;
}

// MXFP4 codes [rows][K/2] as a uint8 matrix read by the W4A4 product: boxes of
// {cb bytes x box_rows}, cb-byte swizzle (cb = 64 or 128), rows and bytes past
// the matrix read as zero.
int encode_gemm_map(const void *codes, int64_t rows, int64_t K, int cb, int box_rows, CUtensorMap *map)
{
    EncodeTiledFn enc;
    int rc = encode_fn(&enc);
    if (rc != KQ_OK) return rc;
    const cuuint64_t dims[2] = {cuuint64_t(K / 2), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(K / 2)};
    const cuuint32_t box[2] = {cuuint32_t(cb), cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           cb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return KQ_OK;
}

// The bf16 output D [M][N] of the W4A4 product: boxes of {box_cols x 32 rows}
// (part of one epilogue warp's row segment), 128-byte swizzle for 64 columns,
// 64-byte swizzle for 32.
int encode_gemm_out_map(void *out, int64_t M, int64_t N, int box_cols, CUtensorMap *map)
{
    EncodeTiledFn enc;
    int rc = encode_fn(&enc);
    if (rc != KQ_OK) return rc;
    const cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(M)};
    const cuuint64_t strides[1] = {cuuint64_t(N) * 2};
    const cuuint32_t box[2] = {cuuint32_t(box_cols), 32};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return KQ_OK;
}

// The scale units of an MXFP4 matrix in the scale-factor layout (row group
// g's units contiguous, 512 bytes each) as a 3-D uint8 tensor {256 bytes,
// 2 Ka half-units, row groups}; boxes of {256, 4, groups}: the two units of a
// 256-element k-chunk for `groups` consecutive row groups.  Units past K and
// row groups past the matrix read as zero.
int encode_sf_map(const void *sf, int64_t rows, int64_t K, int groups, CUtensorMap *map)
{
    EncodeTiledFn enc;
    int rc = encode_fn(&enc);
    if (rc != KQ_OK) return rc;
    const int64_t Ka = (K + 127) / 128;
    const cuuint64_t dims[3] = {256, cuuint64_t(2 * Ka), cuuint64_t((rows + 127) / 128)};
    const cuuint64_t strides[2] = {256, cuuint64_t(Ka) * 512};
    const cuuint32_t box[3] = {256, 4, cuuint32_t(groups)};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(sf), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return KQ_OK;
}

int64_t sf_bytes_of(int64_t rows, int64_t nb) { return ((rows + 127) / 128) * ((nb + 3) / 4) * 512; }

// Default clock budget of a bounded wait: 2^31 cycles, about a second.
constexpr long long kWaitBudget = 1LL << 31;

// Largest block count the staged path takes (row coordinates are int32).
constexpr int64_t kStagedMaxBlocks = (int64_t(1) << 31) - kStageRows;

template <typename Kernel>
int launch_pinned(const char *fn, KernelId id, Kernel kernel, int64_t M, int64_t nb, Geometry *geo)
{
    int64_t target = 0;
    int rc = resident_threads(id, reinterpret_cast<const void *>(kernel), &target);
    if (rc != KQ_OK) return rc;
    *geo = pinned_geometry(M, nb, target);
    (void)fn;
    return KQ_OK;
}

// Grid of the two-block ring kernel (variant 9): one CTA per SM, G a
// multiple of q = nb / gcd(nb, P) so that G * P is a multiple of nb and a
// thread's column never changes (any G with shared factors), at most the SM
// count and no more than the chunks need.  0 where no such G fits.
unsigned ring_grid(int64_t nchunks, int64_t nb, int shared, int P, int sms)
{
    const int64_t q = shared ? 1 : nb / gcd64(nb, P);
    if (q > sms) return 0;
    int64_t G = (sms / q) * q;
    const int64_t need = ((nchunks + q - 1) / q) * q;
    if (G > need) G = need;
    return unsigned(G);
}

// Launch of the ring kernel with P consumers; *launched = false (and KQ_OK)
// where its grid rule or its int32 row coordinates rule the shape out, and
// the caller then runs variant 2.
template <int P>
int ring_launch(const char *fn, KernelId id, const void *act, const float *factors, int shared, uint8_t *codes,
                uint8_t *scales, int64_t nblocks, int64_t nb, cudaStream_t stream, bool *launched)
{
    using C = ring::Cfg<P>;
    *launched = false;
    if (nblocks > int64_t(INT32_MAX) - 2 * P) return KQ_OK;
    int sms = 0;
    int rc = sm_count(&sms);
    if (rc != KQ_OK) return rc;
    const int64_t nchunks = (nblocks + P - 1) / P;
    const unsigned grid = ring_grid(nchunks, nb, shared, P, sms);
    if (grid == 0) return KQ_OK;
    auto k = ring::kq_ring_kernel<P>;
    if ((rc = smem_prepare(id, reinterpret_cast<const void *>(k), C::kSmem)) != KQ_OK) return rc;
    CUtensorMap map;
    if ((rc = encode_act_map(act, nblocks, &map, C::kBoxRows)) != KQ_OK) return rc;
    launch(k, grid, C::kThreads, C::kSmem, stream, map, static_cast<const uint4 *>(act), factors, shared,
                                               reinterpret_cast<uint4 *>(codes), scales, nblocks, int(nb),
                                               kWaitBudget);
    *launched = true;
    return launch_check(fn);
}

// Kernel variants of the KroQuant quantizer: 1 = one block per thread, direct
// 2x2 stages; 2 = packed pairs with the unit-diagonal split, register
// prefetch; 3 = the arithmetic of 2 on TMA-staged input; 4 = the transform
// as tcgen05 MMAs on K split into three bf16 parts; 9 = the operations of 2
// on two rows per thread from a TMA ring.  0 = the default, the fastest on
// the benchmark shapes (2: every form shares the FMA-pipe floor of seven
// lane operations per element, and 2 hides its latency best).
constexpr int kDefaultVariant = 2;

int kq_launch(const char *fn, int variant, const void *act, const float *factors, int shared,
              uint8_t *codes, uint8_t *scales, float *y, bool f32, int64_t M, int64_t d, cudaStream_t stream)
{
    int rc = f32 ? check_quant_args(fn, act, factors, true, y, y, M, d)
                 : check_quant_args(fn, act, factors, true, codes, scales, M, d);
    if (rc == 1) return ok();
    if (rc != KQ_OK) return rc;
    if (variant == 0) variant = kDefaultVariant;
    if (variant < 1 || variant > 9 || (variant >= 5 && variant <= 8))
        return fail(KQ_ERR_VARIANT, "%s: variant %d is not available in this build", fn, variant);
    if (variant == 9 && !f32) {
        const int64_t nb9 = d / kBlk;
        bool launched = false;
        rc = ring_launch<256>(fn, kKqRing, act, factors, shared, codes, scales, M * nb9, nb9, stream, &launched);
        if (rc != KQ_OK || launched) return rc;
    }
    if (variant == 9) variant = 2;   // the fp32 export, or a shape the ring's grid rule excludes
    if (variant == 4 && M < (int64_t(1) << 31)) {
        const int64_t nb4 = d / kBlk;
        CUtensorMap map;
        if ((rc = encode_act_map_rows(act, M, d, &map)) != KQ_OK) return rc;
        const int64_t tiles = ((M + mma::kRows - 1) / mma::kRows) * ((nb4 + mma::kNC - 1) / mma::kNC);
        int sms = 0;
        if ((rc = sm_count(&sms)) != KQ_OK) return rc;
        const unsigned grid = unsigned(tiles < sms ? tiles : sms);
        const float4 *f4 = reinterpret_cast<const float4 *>(factors);
        if (f32) {
            auto k = mma::kq_mma_kernel<KqOut::kF32>;
            if ((rc = mma_prepare(kKqMmaF32, reinterpret_cast<const void *>(k))) != KQ_OK) return rc;
            // the codes map is unused by the fp32 export; any valid map will do
            launch(k, grid, mma::kThreads, mma::kSmem, stream, map, map, f4, shared, nullptr,
                                                           reinterpret_cast<float4 *>(y), M, int(nb4), kWaitBudget);
        } else {
            CUtensorMap cmap;
            if ((rc = encode_codes_map(codes, M, d, &cmap)) != KQ_OK) return rc;
            auto k = mma::kq_mma_kernel<KqOut::kCodes>;
            if ((rc = mma_prepare(kKqMma, reinterpret_cast<const void *>(k))) != KQ_OK) return rc;
            launch(k, grid, mma::kThreads, mma::kSmem, stream, map, cmap, f4, shared, scales, nullptr, M, int(nb4),
                                                           kWaitBudget);
        }
        return launch_check(fn);
    }
    if (variant == 4) variant = 2;   // row coordinates beyond int32: the butterfly
    // the fp32 export and very large inputs use the variant-2 kernel (same arithmetic as 3)
    if (variant == 3 && (f32 || M * (d / kBlk) > kStagedMaxBlocks)) variant = 2;
    const int64_t nb = d / kBlk;
    const int64_t nblocks = M * nb;
    const uint4 *a = static_cast<const uint4 *>(act);
    const float4 *f = reinterpret_cast<const float4 *>(factors);
    Geometry geo;
    if (variant == 3) {
        CUtensorMap map;
        if ((rc = encode_act_map(act, nblocks, &map)) != KQ_OK) return rc;
        int64_t resident = 0;
        if ((rc = staged_prepare(kKqStaged, reinterpret_cast<const void *>(kq_staged_kernel), &resident)) != KQ_OK)
            return rc;
        launch(kq_staged_kernel, staged_grid(nblocks, nb, resident), kStagedThreads, kStagedSmem, stream,
            map, a, f, shared, reinterpret_cast<uint4 *>(codes), scales, nblocks, int(nb), kWaitBudget, 1);
    } else if (variant == 1) {
        if (f32) {
            auto k = kq_butterfly_kernel<KqOut::kF32>;
            if ((rc = launch_pinned(fn, kKqDirectF32, k, M, nb, &geo)) != KQ_OK) return rc;
            launch(k, geo.grid, kThreads, 0, stream, a, f, shared, nullptr, nullptr, reinterpret_cast<float4 *>(y),
                                                 nblocks, int(nb), geo.T);
        } else {
            auto k = kq_butterfly_kernel<KqOut::kCodes>;
            if ((rc = launch_pinned(fn, kKqDirect, k, M, nb, &geo)) != KQ_OK) return rc;
            launch(k, geo.grid, kThreads, 0, stream, a, f, shared, reinterpret_cast<uint4 *>(codes), scales, nullptr,
                                                 nblocks, int(nb), geo.T);
        }
    } else {
        if (f32) {
            auto k = kq_packed_kernel<KqOut::kF32>;
            if ((rc = launch_pinned(fn, kKqPackedF32, k, M, nb, &geo)) != KQ_OK) return rc;
            launch(k, geo.grid, kThreads, 0, stream, a, factors, shared, nullptr, nullptr, reinterpret_cast<float4 *>(y),
                                                 nblocks, int(nb), geo.T);
        } else {
            auto k = kq_packed_kernel<KqOut::kCodes>;
            if ((rc = launch_pinned(fn, kKqPacked, k, M, nb, &geo)) != KQ_OK) return rc;
            launch(k, geo.grid, kThreads, 0, stream, a, factors, shared, reinterpret_cast<uint4 *>(codes), scales, nullptr,
                                                 nblocks, int(nb), geo.T);
        }
    }
    return launch_check(fn);
}

// The W4A4 product, one tile configuration: tensor maps, grid (one CTA per
// SM or per tile), shared-memory attribute (set once per device and
// instantiation), launch.
struct GemmArgs {
    const uint8_t *a_codes, *a_sf, *b_codes, *b_sf;
    void *out;
    bool f32;
    int64_t M, N, K;
    cudaStream_t stream;
};

// Default tile configuration.  Above 128 rows, the SM-pair form: 7 (256 x 256
// tiles) or 8 (256 x 192 tiles), whichever the cost model waves x BN -- rounds
// of one tile per SM pair, each as long as its MMAs -- rates cheaper.  Up to
// 128 rows a pair tile would leave one SM of the pair idle: 4 (256-column
// tiles) or 6 (192-column tiles), whichever waves x (128 + BN) -- rounds of
// one tile per SM, each moving A and B rows -- rates cheaper.
int default_gemm_variant(int64_t M, int64_t N, int sms)
{
    if (M > gemm::kBM) {
        const int64_t pairs = sms / 2 > 0 ? sms / 2 : 1;
        const int64_t mt2 = (M + 2 * gemm::kBM - 1) / (2 * gemm::kBM);
        const int64_t p256 = (mt2 * ((N + 255) / 256) + pairs - 1) / pairs;
        const int64_t p192 = (mt2 * ((N + 191) / 192) + pairs - 1) / pairs;
        return p192 * 192 < p256 * 256 ? 8 : 7;
    }
    const int64_t mt = (M + gemm::kBM - 1) / gemm::kBM;
    const int64_t w256 = (mt * ((N + 255) / 256) + sms - 1) / sms;
    const int64_t w192 = (mt * ((N + 191) / 192) + sms - 1) / sms;
    return w192 * (128 + 192) < w256 * (128 + 256) ? 6 : 4;
}

template <class C, bool F32>
std::atomic<int> g_gemm_smem_set[kMaxDevices];

template <class C, bool F32>
int gemm_launch_out(const GemmArgs &g, const CUtensorMap &amap, const CUtensorMap &bmap, const CUtensorMap &omap,
                    unsigned grid)
{
    auto k = gemm::mxf4_gemm_kernel<C, F32>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices || !g_gemm_smem_set<C, F32>[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmem));
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        if (dev >= 0 && dev < kMaxDevices) g_gemm_smem_set<C, F32>[dev].store(1, std::memory_order_release);
    }
    launch(k, grid, gemm::kThreads, C::kSmem, g.stream, amap, bmap, omap, g.a_sf, g.b_sf, g.out, int(g.M), int(g.N),
                                                     int(g.K), kWaitBudget);
    return launch_check("mxf4_gemm");
}

template <class C>
int gemm_launch(const GemmArgs &g)
{
    const int64_t tiles = ((g.M + gemm::kBM - 1) / gemm::kBM) * ((g.N + C::kBN - 1) / C::kBN);
    if (tiles >= (int64_t(1) << 31)) return fail(KQ_ERR_SHAPE, "mxf4_gemm: too many output tiles");
    CUtensorMap amap, bmap, omap;
    int rc = encode_gemm_map(g.a_codes, g.M, g.K, C::kCB, gemm::kBM, &amap);
    if (rc != KQ_OK) return rc;
    if ((rc = encode_gemm_map(g.b_codes, g.N, g.K, C::kCB, C::kBN, &bmap)) != KQ_OK) return rc;
    // only the TMA-store epilogue reads the output map; the others get a placeholder
    if (C::kTmaOut && !g.f32) {
        if ((rc = encode_gemm_out_map(g.out, g.M, g.N, C::kBN == 256 ? 64 : 32, &omap)) != KQ_OK) return rc;
    } else {
        omap = amap;
    }
    int sms = 0;
    if ((rc = sm_count(&sms)) != KQ_OK) return rc;
    const unsigned grid = unsigned(tiles < sms ? tiles : sms);
    return g.f32 ? gemm_launch_out<C, true>(g, amap, bmap, omap, grid) : gemm_launch_out<C, false>(g, amap, bmap, omap, grid);
}

// The SM-pair form: clusters of two CTAs, as many as fit at once (one CTA
// per SM), each walking 256 x BN tiles.
template <class C, bool F32>
std::atomic<int> g_pair_clusters[kMaxDevices];

template <class C, bool F32>
int gemm_pair_launch_out(const GemmArgs &g, const CUtensorMap *maps, int64_t tiles)
{
    auto k = gemm::mxf4_gemm_pair_kernel<C, F32>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    int clusters = (dev >= 0 && dev < kMaxDevices) ? g_pair_clusters<C, F32>[dev].load(std::memory_order_acquire) : 0;
    if (clusters <= 0) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmem));
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        int sms = 0;
        int rc = sm_count(&sms);
        if (rc != KQ_OK) return rc;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(unsigned(sms / 2 * 2), 1, 1);
        cfg.blockDim = dim3(gemm::kThreads, 1, 1);
        cfg.dynamicSmemBytes = C::kSmem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&clusters, k, &cfg);
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cluster occupancy query: %s", cudaGetErrorString(e));
        if (clusters <= 0) return fail(KQ_ERR_CUDA, "mxf4_gemm: no SM pair can hold the kernel");
        if (dev >= 0 && dev < kMaxDevices) g_pair_clusters<C, F32>[dev].store(clusters, std::memory_order_release);
    }
    const unsigned grid = 2u * unsigned(tiles < clusters ? tiles : clusters);
    launch(k, grid, gemm::kThreads, C::kSmem, g.stream, maps[0], maps[1], maps[2], maps[3], maps[4], g.out, int(g.M),
                                                     int(g.N), int(g.K), kWaitBudget);
    return launch_check("mxf4_gemm");
}

template <class C>
int gemm_pair_launch(const GemmArgs &g)
{
    const int64_t tiles = ((g.M + 2 * gemm::kBM - 1) / (2 * gemm::kBM)) * ((g.N + C::kBN - 1) / C::kBN);
    if (tiles >= (int64_t(1) << 31)) return fail(KQ_ERR_SHAPE, "mxf4_gemm: too many output tiles");
    CUtensorMap maps[5];   // A codes, B codes, A scales, B scales, D
    int rc = encode_gemm_map(g.a_codes, g.M, g.K, C::kCB, gemm::kBM, &maps[0]);
    if (rc != KQ_OK) return rc;
    if ((rc = encode_gemm_map(g.b_codes, g.N, g.K, C::kCB, C::kBRows, &maps[1])) != KQ_OK) return rc;
    if ((rc = encode_sf_map(g.a_sf, g.M, g.K, 1, &maps[2])) != KQ_OK) return rc;
    if ((rc = encode_sf_map(g.b_sf, g.N, g.K, 2, &maps[3])) != KQ_OK) return rc;
    // only the bf16 epilogue reads the output map ({32 x 32} boxes); fp32 gets a placeholder
    if (!g.f32) {
        if ((rc = encode_gemm_out_map(g.out, g.M, g.N, 32, &maps[4])) != KQ_OK) return rc;
    } else {
        maps[4] = maps[0];
    }
    return g.f32 ? gemm_pair_launch_out<C, true>(g, maps, tiles) : gemm_pair_launch_out<C, false>(g, maps, tiles);
}

// Shared memory of the long-row kernel: the (1 + gamma, beta) table, the
// row ring and the reduction arrays.
size_t cols_smem(int nt, int depth) { return size_t(16) * nt * 16 + size_t(depth) * nt * 64 + size_t(nt / 32) * 48; }

template <bool SF, int DEPTH, int MAXT>
int cols_launch(const char *fn, const void *h_bf16, const float *gamma, const float *beta, int64_t nsamples,
                float eps, const float *factors, int shared, uint8_t *out_codes, uint8_t *out_scales, int64_t M,
                int nb, int sms, cudaStream_t stream)
{
    const int nt = (nb + 31) / 32 * 32;
    const size_t smem = cols_smem(nt, DEPTH);
    auto k = norm_kq_cols_kernel<SF, DEPTH, MAXT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, nt, smem);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
    if (per_sm < 1) return fail(KQ_ERR_CUDA, "%s: the long-row kernel does not fit on this device", fn);
    const int64_t rows_per = M / nsamples;
    int64_t cps = int64_t(sms) * per_sm / nsamples;
    if (cps > rows_per) cps = rows_per;
    if (cps < 1) cps = 1;
    if (cps * nsamples >= (int64_t(1) << 31)) cps = ((int64_t(1) << 31) - 1) / nsamples;
    launch(k, unsigned(cps * nsamples), nt, smem, stream, static_cast<const uint4 *>(h_bf16), gamma, beta, rows_per, eps,
                                                      factors, shared ? 1 : 0, reinterpret_cast<uint4 *>(out_codes),
                                                      out_scales, nb, int(cps));
    return launch_check(fn);
}

// Kernels of the fused normalisation: 1 = the single-pass row kernel (where
// a configuration fits), 2 = the warp-per-row kernel that re-reads the row,
// 3 = the long-row kernel; 0 = the default: 3 from kColsMinBlocks block
// columns up (d >= 6144), else 1 where it fits, else 2.
constexpr int kColsMinBlocks = 192;

template <bool SF>
int norm_launch(const char *fn, const void *h_bf16, const float *gamma, const float *beta, int64_t nsamples, float eps,
                const float *factors, int shared, uint8_t *out_codes, uint8_t *out_scales, int64_t M, int64_t d,
                cudaStream_t stream, int variant = 0)
{
    if (M < 0 || d <= 0 || d % kBlk != 0 || d / kBlk > 512)
        return fail(KQ_ERR_SHAPE, "%s: need M >= 0 and d a positive multiple of 32, at most 16384 (M=%lld, d=%lld)",
                    fn, (long long)M, (long long)d);
    if (nsamples <= 0 || M % nsamples != 0)
        return fail(KQ_ERR_SHAPE, "%s: M must be a multiple of nsamples > 0 (M=%lld, nsamples=%lld)", fn,
                    (long long)M, (long long)nsamples);
    if (M > 0 && M > INT64_MAX / d) return fail(KQ_ERR_SHAPE, "%s: size too large", fn);
    if (!(eps >= 0.0f)) return fail(KQ_ERR_SHAPE, "%s: eps must be >= 0", fn);
    if (M == 0) return ok();
    if (!h_bf16 || !gamma || !beta || !factors || !out_codes || !out_scales)
        return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    if (!aligned(h_bf16, 16) || !aligned(out_codes, 16) || !aligned(factors, 16) || !aligned(gamma, 16) ||
        !aligned(beta, 16))
        return fail(KQ_ERR_ALIGN, "%s: h, out_codes, factors, gamma and beta must be 16-byte aligned", fn);
    if (variant < 0 || variant > 3)
        return fail(KQ_ERR_VARIANT, "%s: variant %d is not available in this build", fn, variant);
    const int nb = int(d / kBlk);
    int sms = 0;
    int rc = sm_count(&sms);
    if (rc != KQ_OK) return rc;
    if (variant == 0) variant = nb >= kColsMinBlocks ? 3 : 1;
    if (variant == 3) {
        // up to 384 threads (d <= 12288): a 4-row ring (two pairs) and up to 168
        // registers; wider rows: 512 threads, a 2-row ring, 128 registers
        if (nb <= 384)
            return cols_launch<SF, 4, 384>(fn, h_bf16, gamma, beta, nsamples, eps, factors, shared, out_codes,
                                           out_scales, M, nb, sms, stream);
        return cols_launch<SF, 2, 512>(fn, h_bf16, gamma, beta, nsamples, eps, factors, shared, out_codes, out_scales,
                                       M, nb, sms, stream);
    }
    if (variant == 1) {
        // single-pass kernel: the first (warps, row buffers) whose shared memory
        // fits, chosen once per device and row width (cached: warps << 8 | nbuf
        // << 4 | CTAs per SM; -1 = none fits)
        int devc = 0;
        cudaError_t e2 = cudaGetDevice(&devc);
        if (e2 != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e2));
        const size_t tab = size_t(nb) * kNormRowSlot * 16, row = size_t(nb) * 64;
        int packed = (devc >= 0 && devc < kMaxDevices) ? g_norm_cfg[SF][devc][nb].load(std::memory_order_acquire) : 0;
        if (packed == 0) {
            packed = -1;
            e2 = cudaFuncSetAttribute(norm_kq_rows_kernel<SF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(kNormRowsSmemMax));
            if (e2 != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e2));
            // fewer than 4 row buffers per CTA would leave the SM nearly idle: the
            // fallback kernel is then faster
            const int cfg[8][2] = {{16, 2}, {16, 1}, {8, 2}, {12, 1}, {4, 2}, {8, 1}, {2, 2}, {4, 1}};
            for (const auto &c : cfg) {
                const size_t smem_r = tab + size_t(c[0]) * c[1] * row;
                if (smem_r > kNormRowsSmemMax) continue;
                int per_sm = 0;
                e2 = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, norm_kq_rows_kernel<SF>, 32 * c[0], smem_r);
                if (e2 != cudaSuccess) return fail(KQ_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e2));
                if (per_sm < 1) continue;
                packed = (c[0] << 8) | (c[1] << 4) | (per_sm > 15 ? 15 : per_sm);
                break;
            }
            if (devc >= 0 && devc < kMaxDevices) g_norm_cfg[SF][devc][nb].store(packed, std::memory_order_release);
        }
        if (packed > 0) {
            const int warps = packed >> 8, nbuf = (packed >> 4) & 15, per_sm = packed & 15;
            const int64_t rows_per = M / nsamples;
            int64_t cps = int64_t(sms) * per_sm / nsamples;
            const int64_t most = rows_per / warps;          // at least one row per warp per CTA
            if (cps > most) cps = most;
            if (cps < 1) cps = 1;
            if (cps * nsamples >= (int64_t(1) << 31)) cps = ((int64_t(1) << 31) - 1) / nsamples;
            const size_t smem_r = tab + size_t(warps) * nbuf * row;
            launch(norm_kq_rows_kernel<SF>, unsigned(cps * nsamples), 32 * warps, smem_r, stream,
                static_cast<const uint4 *>(h_bf16), gamma, beta, rows_per, eps, factors, shared ? 1 : 0,
                reinterpret_cast<uint4 *>(out_codes), out_scales, nb, int(cps), nbuf);
            return launch_check(fn);
        }
    }
    const size_t smem = size_t(nb) * kNormSlot * sizeof(float);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (smem > 48 * 1024 && (dev < 0 || dev >= kMaxDevices || !g_smem_set[SF ? kNormKqSf : kNormKq][dev].load())) {
        e = cudaFuncSetAttribute(norm_kq_kernel<SF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(size_t(512) * kNormSlot * sizeof(float)));
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        if (dev >= 0 && dev < kMaxDevices) g_smem_set[SF ? kNormKqSf : kNormKq][dev].store(1);
    }
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, norm_kq_kernel<SF>, kThreads, smem);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
    if (per_sm < 1) per_sm = 1;
    const int64_t warps_needed = M;
    int64_t grid = int64_t(sms) * per_sm;
    const int64_t need = (warps_needed + (kThreads / 32) - 1) / (kThreads / 32);
    if (grid > need) grid = need;
    launch(norm_kq_kernel<SF>, unsigned(grid), kThreads, smem, stream,
        static_cast<const uint4 *>(h_bf16), gamma, beta, M / nsamples, eps, factors, shared ? 1 : 0,
        reinterpret_cast<uint4 *>(out_codes), out_scales, M, nb);
    return launch_check(fn);
}

}  // namespace

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" {

int kq_abi_version(void) { return 1; }

const char *kq_last_error(void) { return tl_err; }

int kq_quantize(const void *act_bf16, const float *factors, uint8_t *out_codes, uint8_t *out_scales, int64_t M,
                int64_t d, cudaStream_t stream)
{
    return kq_launch("kq_quantize", 0, act_bf16, factors, 0, out_codes, out_scales, nullptr, false, M, d, stream);
}

int kq_quantize_shared(const void *act_bf16, const float *factors, uint8_t *out_codes, uint8_t *out_scales,
                       int64_t M, int64_t d, cudaStream_t stream)
{
    return kq_launch("kq_quantize_shared", 0, act_bf16, factors, 1, out_codes, out_scales, nullptr, false, M, d,
                     stream);
}

int kq_quantize_variant(int variant, const void *act_bf16, const float *factors, int shared, uint8_t *out_codes,
                        uint8_t *out_scales, int64_t M, int64_t d, cudaStream_t stream)
{
    return kq_launch("kq_quantize_variant", variant, act_bf16, factors, shared ? 1 : 0, out_codes, out_scales,
                     nullptr, false, M, d, stream);
}

int kq_transform_f32_variant(int variant, const void *act_bf16, const float *factors, int shared, float *out_y,
                             int64_t M, int64_t d, cudaStream_t stream)
{
    return kq_launch("kq_transform_f32_variant", variant, act_bf16, factors, shared ? 1 : 0, nullptr, nullptr, out_y,
                     true, M, d, stream);
}

int kq_transform_f32(const void *act_bf16, const float *factors, int shared, float *out_y, int64_t M, int64_t d,
                     cudaStream_t stream)
{
    return kq_launch("kq_transform_f32", 0, act_bf16, factors, shared ? 1 : 0, nullptr, nullptr, out_y, true, M, d,
                     stream);
}

int sq_quantize(const void *act_bf16, const float *mult, uint8_t *out_codes, uint8_t *out_scales, int64_t M,
                int64_t d, cudaStream_t stream)
{
    return sq_quantize_variant(0, act_bf16, mult, out_codes, out_scales, M, d, stream);
}

int mx_quantize(const void *act_bf16, uint8_t *out_codes, uint8_t *out_scales, int64_t M, int64_t d,
                cudaStream_t stream)
{
    return mx_quantize_variant(0, act_bf16, out_codes, out_scales, M, d, stream);
}

int sq_quantize_variant(int variant, const void *act_bf16, const float *mult, uint8_t *out_codes,
                        uint8_t *out_scales, int64_t M, int64_t d, cudaStream_t stream)
{
    const char *fn = "sq_quantize";
    int rc = check_quant_args(fn, act_bf16, mult, true, out_codes, out_scales, M, d);
    if (rc == 1) return ok();
    if (rc != KQ_OK) return rc;
    if (variant == 0) variant = 2;
    if (variant != 1 && variant != 2)
        return fail(KQ_ERR_VARIANT, "%s: variant %d is not available in this build", fn, variant);
    const int64_t nb = d / kBlk;
    const int64_t nblocks = M * nb;
    if (variant == 2 && nblocks <= kStagedMaxBlocks) {
        CUtensorMap map;
        if ((rc = encode_act_map(act_bf16, nblocks, &map)) != KQ_OK) return rc;
        int64_t resident = 0;
        if ((rc = staged_prepare(kSqStaged, reinterpret_cast<const void *>(sq_staged_kernel), &resident)) != KQ_OK)
            return rc;
        launch(sq_staged_kernel, staged_grid(nblocks, nb, resident), kStagedThreads, kStagedSmem, stream,
            map, reinterpret_cast<const float4 *>(mult), reinterpret_cast<uint4 *>(out_codes), out_scales, nblocks,
            int(nb), kWaitBudget, 1);
        return launch_check(fn);
    }
    Geometry geo;
    if ((rc = launch_pinned(fn, kSqPacked, sq_packed_kernel, M, nb, &geo)) != KQ_OK) return rc;
    launch(sq_packed_kernel, geo.grid, kThreads, 0, stream, static_cast<const uint4 *>(act_bf16),
                                                        reinterpret_cast<const float4 *>(mult),
                                                        reinterpret_cast<uint4 *>(out_codes), out_scales, nblocks,
                                                        int(nb), geo.T);
    return launch_check(fn);
}

int mx_quantize_variant(int variant, const void *act_bf16, uint8_t *out_codes, uint8_t *out_scales, int64_t M,
                        int64_t d, cudaStream_t stream)
{
    const char *fn = "mx_quantize";
    int rc = check_quant_args(fn, act_bf16, nullptr, false, out_codes, out_scales, M, d);
    if (rc == 1) return ok();
    if (rc != KQ_OK) return rc;
    if (variant == 0) variant = 1;   // register prefetch: 4 CTAs/SM hide the latency already
    if (variant != 1 && variant != 2)
        return fail(KQ_ERR_VARIANT, "%s: variant %d is not available in this build", fn, variant);
    const int64_t nb = d / kBlk;
    const int64_t nblocks = M * nb;
    if (variant == 2 && nblocks <= kStagedMaxBlocks) {
        CUtensorMap map;
        if ((rc = encode_act_map(act_bf16, nblocks, &map)) != KQ_OK) return rc;
        int64_t resident = 0;
        if ((rc = staged_prepare(kMxStaged, reinterpret_cast<const void *>(mx_staged_kernel), &resident)) != KQ_OK)
            return rc;
        // any grid works for MX (no per-column state); keep the same sizing
        launch(mx_staged_kernel, staged_grid(nblocks, 1, resident), kStagedThreads, kStagedSmem, stream,
            map, reinterpret_cast<uint4 *>(out_codes), out_scales, nblocks, kWaitBudget, 1);
        return launch_check(fn);
    }
    Geometry geo;
    if ((rc = launch_pinned(fn, kMxPacked, mx_packed_kernel, M, nb, &geo)) != KQ_OK) return rc;
    launch(mx_packed_kernel, geo.grid, kThreads, 0, stream, static_cast<const uint4 *>(act_bf16),
                                                        reinterpret_cast<uint4 *>(out_codes), out_scales, nblocks,
                                                        geo.T);
    return launch_check(fn);
}

int kq_quantize_lu(const void *act_bf16, const float *lu_params, int shared, uint8_t *out_codes,
                   uint8_t *out_scales, int64_t M, int64_t d, cudaStream_t stream)
{
    const char *fn = "kq_quantize_lu";
    if (M < 0 || d <= 0 || d % kBlk != 0)
        return fail(KQ_ERR_SHAPE, "%s: need M >= 0 and d a positive multiple of 32 (M=%lld, d=%lld)", fn,
                    (long long)M, (long long)d);
    if (d / kBlk > INT32_MAX || (M > 0 && M > INT64_MAX / d))
        return fail(KQ_ERR_SHAPE, "%s: size too large", fn);
    if (M == 0) return ok();
    if (!act_bf16 || !lu_params || !out_codes || !out_scales) return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    if (!aligned(act_bf16, 16) || !aligned(out_codes, 16) || !aligned(lu_params, 4))
        return fail(KQ_ERR_ALIGN, "%s: act and out_codes must be 16-byte aligned, lu_params 4-byte", fn);
    const int64_t nb = d / kBlk;
    Geometry geo;
    auto k = kq_packed_kernel<KqOut::kCodes, true>;
    int rc = launch_pinned(fn, kKqLu, k, M, nb, &geo);
    if (rc != KQ_OK) return rc;
    launch(k, geo.grid, kThreads, 0, stream, static_cast<const uint4 *>(act_bf16), lu_params, shared ? 1 : 0,
                                         reinterpret_cast<uint4 *>(out_codes), out_scales, nullptr, M * nb, int(nb),
                                         geo.T);
    return launch_check(fn);
}

int fwht_quantize(const void *act_bf16, int64_t H, uint8_t *out_codes, uint8_t *out_scales, int64_t M, int64_t d,
                  cudaStream_t stream)
{
    const char *fn = "fwht_quantize";
    int xstages = -1;
    for (int s = 0; s <= 5; ++s)
        if (H == (int64_t(32) << s)) xstages = s;
    if (xstages < 0) return fail(KQ_ERR_SHAPE, "%s: H must be a power of two in [32, 1024] (H=%lld)", fn, (long long)H);
    if (M < 0 || d <= 0 || d % H != 0)
        return fail(KQ_ERR_SHAPE, "%s: need M >= 0 and d a positive multiple of H (M=%lld, d=%lld, H=%lld)", fn,
                    (long long)M, (long long)d, (long long)H);
    if (d / kBlk > INT32_MAX || (M > 0 && M > INT64_MAX / d))
        return fail(KQ_ERR_SHAPE, "%s: size too large", fn);
    if (M == 0) return ok();
    if (!act_bf16 || !out_codes || !out_scales) return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    if (!aligned(act_bf16, 16) || !aligned(out_codes, 16))
        return fail(KQ_ERR_ALIGN, "%s: act and out_codes must be 16-byte aligned", fn);
    const int64_t nblocks = M * (d / kBlk);
    int64_t target = 0;
    int rc = resident_threads(kFwht, reinterpret_cast<const void *>(fwht_kernel), &target);
    if (rc != KQ_OK) return rc;
    int64_t T = (target / 32) * 32;
    const int64_t need = ((nblocks + 31) / 32) * 32;
    if (T > need) T = need;
    if (T < 32) T = 32;
    const unsigned grid = unsigned((T + kThreads - 1) / kThreads);
    // 1/sqrt(H) rounded to fp32: H = 2^(5 + s); sqrt(2^n) = 2^(n/2) * (sqrt 2 if n odd)
    const double inv = 1.0 / std::sqrt(double(H));
    launch(fwht_kernel, grid, kThreads, 0, stream, static_cast<const uint4 *>(act_bf16),
                                               reinterpret_cast<uint4 *>(out_codes), out_scales, nblocks,
                                               int64_t(grid) * kThreads, xstages, float(inv));
    return launch_check(fn);
}

int kq_inverse_f32(const float *y, const float *factors, int shared, float *x_out, int64_t M, int64_t d,
                   cudaStream_t stream)
{
    const char *fn = "kq_inverse_f32";
    if (M < 0 || d <= 0 || d % kBlk != 0) return fail(KQ_ERR_SHAPE, "%s: need M >= 0 and d a positive multiple of 32", fn);
    if (d / kBlk > INT32_MAX || (M > 0 && M > INT64_MAX / d)) return fail(KQ_ERR_SHAPE, "%s: size too large", fn);
    if (M == 0) return ok();
    if (!y || !factors || !x_out) return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    if (!aligned(y, 16) || !aligned(x_out, 16) || !aligned(factors, 16))
        return fail(KQ_ERR_ALIGN, "%s: y, x_out and factors must be 16-byte aligned", fn);
    const int64_t nb = d / kBlk;
    Geometry geo;
    int rc = launch_pinned(fn, kInverse, fold_kernel<true>, M, nb, &geo);
    if (rc != KQ_OK) return rc;
    launch(fold_kernel<true>, geo.grid, kThreads, 0, stream, reinterpret_cast<const float4 *>(y),
                                                         reinterpret_cast<const float4 *>(factors), shared ? 1 : 0,
                                                         reinterpret_cast<float4 *>(x_out), M * nb, int(nb), geo.T);
    return launch_check(fn);
}

int mx_dequantize(const uint8_t *codes, const uint8_t *scales, float *out, int64_t M, int64_t d, cudaStream_t stream)
{
    const char *fn = "mx_dequantize";
    if (M < 0 || d <= 0 || d % kBlk != 0) return fail(KQ_ERR_SHAPE, "%s: need M >= 0 and d a positive multiple of 32", fn);
    if (d / kBlk > INT32_MAX || (M > 0 && M > INT64_MAX / d)) return fail(KQ_ERR_SHAPE, "%s: size too large", fn);
    if (M == 0) return ok();
    if (!codes || !scales || !out) return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    if (!aligned(codes, 16) || !aligned(out, 16)) return fail(KQ_ERR_ALIGN, "%s: codes and out must be 16-byte aligned", fn);
    const int64_t nblocks = M * (d / kBlk);
    int64_t target = 0;
    int rc = resident_threads(kDequant, reinterpret_cast<const void *>(mx_dequantize_kernel), &target);
    if (rc != KQ_OK) return rc;
    int64_t T = target < nblocks ? target : nblocks;
    launch(mx_dequantize_kernel, unsigned((T + kThreads - 1) / kThreads), kThreads, 0, stream,
        reinterpret_cast<const uint4 *>(codes), scales, reinterpret_cast<float4 *>(out), nblocks);
    return launch_check(fn);
}

int norm_kq_quantize(const void *h_bf16, const float *gamma, const float *beta, int64_t nsamples, float eps,
                     const float *factors, int shared, uint8_t *out_codes, uint8_t *out_scales, int64_t M, int64_t d,
                     cudaStream_t stream)
{
    return norm_launch<false>("norm_kq_quantize", h_bf16, gamma, beta, nsamples, eps, factors, shared, out_codes,
                              out_scales, M, d, stream);
}

int norm_kq_quantize_sf(const void *h_bf16, const float *gamma, const float *beta, int64_t nsamples, float eps,
                        const float *factors, int shared, uint8_t *out_codes, uint8_t *out_sf, int64_t M, int64_t d,
                        cudaStream_t stream)
{
    return norm_launch<true>("norm_kq_quantize_sf", h_bf16, gamma, beta, nsamples, eps, factors, shared, out_codes,
                             out_sf, M, d, stream);
}

int norm_kq_quantize_variant(int variant, const void *h_bf16, const float *gamma, const float *beta,
                             int64_t nsamples, float eps, const float *factors, int shared, uint8_t *out_codes,
                             uint8_t *out_scales, int64_t M, int64_t d, cudaStream_t stream)
{
    return norm_launch<false>("norm_kq_quantize_variant", h_bf16, gamma, beta, nsamples, eps, factors, shared,
                              out_codes, out_scales, M, d, stream, variant);
}

int64_t kq_sf_bytes(int64_t rows, int64_t d)
{
    if (rows < 0 || d <= 0 || d % kBlk != 0) return -1;
    return sf_bytes_of(rows, d / kBlk);
}

int kq_quantize_sf(const void *act_bf16, const float *factors, int shared, uint8_t *out_codes, uint8_t *out_sf,
                   int64_t M, int64_t d, cudaStream_t stream)
{
    const char *fn = "kq_quantize_sf";
    int rc = check_quant_args(fn, act_bf16, factors, true, out_codes, out_sf, M, d);
    if (rc == 1) return ok();
    if (rc != KQ_OK) return rc;
    const int64_t nb = d / kBlk;
    Geometry geo;
    auto k = kq_packed_kernel<KqOut::kCodes, false, true>;
    if ((rc = launch_pinned(fn, kKqPackedSf, k, M, nb, &geo)) != KQ_OK) return rc;
    launch(k, geo.grid, kThreads, 0, stream, static_cast<const uint4 *>(act_bf16), factors, shared ? 1 : 0,
                                         reinterpret_cast<uint4 *>(out_codes), out_sf, nullptr, M * nb, int(nb),
                                         geo.T);
    return launch_check(fn);
}

int mx_quantize_f32(const float *x, uint8_t *out_codes, uint8_t *out_scales, int scale_layout, int64_t M, int64_t d,
                    cudaStream_t stream)
{
    const char *fn = "mx_quantize_f32";
    if (scale_layout != KQ_SCALES_ROWMAJOR && scale_layout != KQ_SCALES_SF)
        return fail(KQ_ERR_SHAPE, "%s: scale_layout must be KQ_SCALES_ROWMAJOR or KQ_SCALES_SF", fn);
    int rc = check_quant_args(fn, x, nullptr, false, out_codes, out_scales, M, d);
    if (rc == 1) return ok();
    if (rc != KQ_OK) return rc;
    const int64_t nb = d / kBlk;
    const int64_t nblocks = M * nb;
    const bool sf = scale_layout == KQ_SCALES_SF;
    auto k = sf ? mx_f32_kernel<true> : mx_f32_kernel<false>;
    int64_t target = 0;
    if ((rc = resident_threads(sf ? kMxF32Sf : kMxF32, reinterpret_cast<const void *>(k), &target)) != KQ_OK)
        return rc;
    const int64_t T = target < nblocks ? target : nblocks;
    launch(k, unsigned((T + kThreads - 1) / kThreads), kThreads, 0, stream,
        reinterpret_cast<const float4 *>(x), reinterpret_cast<uint4 *>(out_codes), out_scales, nblocks, int(nb));
    return launch_check(fn);
}

int mx_scales_to_sf(const uint8_t *scales, uint8_t *out_sf, int64_t M, int64_t d, cudaStream_t stream)
{
    const char *fn = "mx_scales_to_sf";
    if (M < 0 || d <= 0 || d % kBlk != 0)
        return fail(KQ_ERR_SHAPE, "%s: need M >= 0 and d a positive multiple of 32", fn);
    if (d / kBlk > INT32_MAX || (M > 0 && M > INT64_MAX / d)) return fail(KQ_ERR_SHAPE, "%s: size too large", fn);
    if (M == 0) return ok();
    if (!scales || !out_sf) return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    const int64_t n = M * (d / kBlk);
    int64_t target = 0;
    int rc = resident_threads(kSfRelayout, reinterpret_cast<const void *>(sf_relayout_kernel), &target);
    if (rc != KQ_OK) return rc;
    const int64_t T = target < n ? target : n;
    launch(sf_relayout_kernel, unsigned((T + kThreads - 1) / kThreads), kThreads, 0, stream, scales, out_sf, n,
                                                                                          int(d / kBlk));
    return launch_check(fn);
}

int mxf4_gemm_variant(int variant, const uint8_t *a_codes, const uint8_t *a_sf, const uint8_t *b_codes,
                      const uint8_t *b_sf, void *out, int out_f32, int64_t M, int64_t N, int64_t K, cudaStream_t stream)
{
    const char *fn = "mxf4_gemm";
    if (M < 0 || N < 0 || K <= 0 || K % kBlk != 0 || N % 8 != 0)
        return fail(KQ_ERR_SHAPE, "%s: need M >= 0, N >= 0 a multiple of 8, K a positive multiple of 32 "
                    "(M=%lld, N=%lld, K=%lld)", fn, (long long)M, (long long)N, (long long)K);
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return fail(KQ_ERR_SHAPE, "%s: M, N and K must be below 2^31", fn);
    if (variant < 0 || variant > 8) return fail(KQ_ERR_VARIANT, "%s: variant %d is not available", fn, variant);
    if (M == 0 || N == 0) return ok();
    if (!a_codes || !a_sf || !b_codes || !b_sf || !out) return fail(KQ_ERR_NULL, "%s: NULL pointer argument", fn);
    if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) ||
        !aligned(out, 16))
        return fail(KQ_ERR_ALIGN, "%s: every pointer must be 16-byte aligned", fn);
    if (variant == 0) {
        int sms = 0;
        int rc = sm_count(&sms);
        if (rc != KQ_OK) return rc;
        variant = default_gemm_variant(M, N, sms);
    }
    const GemmArgs g{a_codes, a_sf, b_codes, b_sf, out, out_f32 != 0, M, N, K, stream};
    switch (variant) {
    case 1: return gemm_launch<gemm::Cfg1>(g);
    case 2: return gemm_launch<gemm::Cfg2>(g);
    case 3: return gemm_launch<gemm::Cfg3>(g);
    case 4: return gemm_launch<gemm::Cfg4>(g);
    case 5: return gemm_launch<gemm::Cfg5>(g);
    case 6: return gemm_launch<gemm::Cfg6>(g);
    case 7: return gemm_pair_launch<gemm::Pair7>(g);
    default: return gemm_pair_launch<gemm::Pair8>(g);
    }
}

int mxf4_gemm(const uint8_t *a_codes, const uint8_t *a_sf, const uint8_t *b_codes, const uint8_t *b_sf, void *out,
              int out_f32, int64_t M, int64_t N, int64_t K, cudaStream_t stream)
{
    return mxf4_gemm_variant(0, a_codes, a_sf, b_codes, b_sf, out, out_f32, M, N, K, stream);
}

int kq_wait_timeouts(int *count, int reset)
{
    if (!count) return fail(KQ_ERR_NULL, "kq_wait_timeouts: NULL pointer argument");
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_wait_timeouts, sizeof v);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "kq_wait_timeouts: %s", cudaGetErrorString(e));
    if (reset) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof zero);
        if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "kq_wait_timeouts: %s", cudaGetErrorString(e));
    }
    *count = v;
    return ok();
}

int kq_selftest_bounded_wait(cudaStream_t stream)
{
    // One CTA whose producer issues no copies: every consumer wait and the
    // producer's own wait run out after ~2^21 cycles (about a millisecond).
    // No memory is read or written besides the counter; the dummy address
    // only has to satisfy the tensor map's alignment rule.
    void *dummy = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&dummy, g_selftest_dummy);
    if (e != cudaSuccess) return fail(KQ_ERR_CUDA, "kq_selftest_bounded_wait: %s", cudaGetErrorString(e));
    const int64_t nblocks = kSelftestBlocks;
    CUtensorMap map;
    int rc = encode_act_map(dummy, nblocks, &map);
    if (rc != KQ_OK) return rc;
    int64_t resident = 0;
    if ((rc = staged_prepare(kMxStaged, reinterpret_cast<const void *>(mx_staged_kernel), &resident)) != KQ_OK)
        return rc;
    launch(mx_staged_kernel, 1, kStagedThreads, kStagedSmem, stream, map, static_cast<uint4 *>(dummy),
                                                                 static_cast<uint8_t *>(dummy), nblocks, 1LL << 21, 0);
    return launch_check("kq_selftest_bounded_wait");
}

int kq_fold_weights(const float *W, const float *factors, int shared, float *W_out, int64_t N, int64_t d,
                    cudaStream_t stream)
{
    if (N < 0 || d <= 0 || d % kBlk != 0)
        return fail(KQ_ERR_SHAPE, "kq_fold_weights: need N >= 0 and d a positive multiple of 32");
    if (d / kBlk > INT32_MAX || (N > 0 && N > INT64_MAX / d))
        return fail(KQ_ERR_SHAPE, "kq_fold_weights: size too large");
    if (N == 0) return ok();
    if (!W || !factors || !W_out) return fail(KQ_ERR_NULL, "kq_fold_weights: NULL pointer argument");
    if (!aligned(W, 16) || !aligned(W_out, 16) || !aligned(factors, 16))
        return fail(KQ_ERR_ALIGN, "kq_fold_weights: W, W_out and factors must be 16-byte aligned");
    const int64_t nb = d / kBlk;
    Geometry geo;
    int rc = launch_pinned("kq_fold_weights", kFold, fold_kernel<false>, N, nb, &geo);
    if (rc != KQ_OK) return rc;
    launch(fold_kernel<false>, geo.grid, kThreads, 0, stream, reinterpret_cast<const float4 *>(W),
                                                   reinterpret_cast<const float4 *>(factors), shared ? 1 : 0,
                                                   reinterpret_cast<float4 *>(W_out), N * nb, int(nb), geo.T);
    return launch_check("kq_fold_weights");
}

}  // extern "C"
