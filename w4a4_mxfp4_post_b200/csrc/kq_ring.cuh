// kq_ring.cuh -- KroQuant quantizer, variant 9: two blocks per thread on a
// TMA ring.  Included by kroquant.cu; uses its helpers (mbarriers, TMA, the
// unit-diagonal split, the MXFP4 pieces).
//
// The transform of the pages (KroQuant section 3.2, Eq. (4): y = (G1 (x) ...
// (x) G5) x per 32-channel block) is applied in the unit-diagonal form of
// variant 2 (K = D U, U = (x)_k [[1, b_k], [c_k, 1]]), with the same
// operations in the same order, so the two variants give bit-identical
// results.  What changes is the data layout and the memory pipeline:
//
// * Two blocks per thread, one register pair per in-block index.  A thread
//   owns one block column j and transforms two of its rows at once: p[i] =
//   (x_i of row r, x_i of row r'), so all five radix-2 stages and the D
//   multiply are packed f32x2 FMAs with broadcast coefficients (variant 2's
//   pair layout (x_i, x_{i+16}) leaves the stage on bit 4 to scalar FMAs).
//   5 x 32 + 32 = 192 packed FMAs per 64 elements, and two independent
//   dependency chains per thread.
// * A ring of kStages shared-memory stages fed by one producer thread with
//   2-D tensor copies (cp.async.bulk.tensor, 64-byte swizzle: the 16-byte
//   chunk q of row r lands at chunk q ^ ((r >> 1) & 3), so the consumers'
//   16-byte shared loads are conflict-free), so the bytes in flight (up to
//   kStages x P x 64 per SM) do not cost registers.  The activation is seen
//   as a [nblocks][32] bf16 matrix, one 64-byte row per block; a stage holds
//   P consecutive blocks (one per consumer thread).
// * One persistent CTA per SM.  CTA b takes the chunks b, b + G, b + 2G, ...
//   (G = gridDim.x) and its consumers take them two at a time; thread t owns
//   row t of every stage, i.e. block c * P + t.  With G * P a multiple of nb
//   (the host picks G so), a thread's column never changes and the two
//   blocks of a step are rows of the same column: the column's 42
//   coefficients (D and the 10 off-diagonal values) are set up once.
//
// Every mbarrier wait is bounded (g_wait_timeouts) and the give-up decision
// is warp-uniform; the producer drains its copies in flight before exiting.

namespace ring {

template <int P>
struct Cfg {
    static constexpr int kConsumers = P;                    // = blocks per stage
    static constexpr int kBoxRows = P > 256 ? P / 2 : P;    // TMA boxes are at most 256 rows
    static constexpr int kBoxes = P / kBoxRows;
    static constexpr int kStageBytes = P * 64;
    static constexpr int kStages = 8;                       // even: a step takes stages s, s + 1
    static constexpr int kThreads = P + 32;                 // + one producer warp
    static constexpr size_t kSmem = size_t(kStages) * kStageBytes + 1024 + 2 * kStages * sizeof(uint64_t);
    static_assert(P % 64 == 0 && kBoxRows <= 256 && kBoxRows * kBoxes == P, "stage geometry");
    static_assert(kStages % 2 == 0, "stages are consumed in pairs");
    static_assert((kBoxRows * 64) % 1024 == 0, "each box keeps the swizzle alignment");
    static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

// The column's coefficients of the unit-diagonal form: D (32 values, element
// i of a block scaled by D[i]) and the off-diagonal coefficients of the five
// unit factors, B[bit], C[bit] for the stage on in-block index bit `bit`
// (bit 4 = G1, bit 0 = G5).
struct Coef {
    float D[32];
    float B[5], C[5];
};

// Same splits and the same D products, in the same order, as kq_fast_setup.
__device__ __forceinline__ bool coef_setup(const float4 (&g)[5], Coef &st)
{
    float d0[5], d1[5], bb[5], cc[5];
    bool fast = true;
#pragma unroll
    for (int k = 0; k < 5; ++k) fast &= unit_split(g[k], d0[k], d1[k], bb[k], cc[k]);
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
    for (int i = 0; i < 32; ++i) st.D[i] = dd[i];
#pragma unroll
    for (int bit = 0; bit < 5; ++bit) {
        st.B[bit] = bb[4 - bit];
        st.C[bit] = cc[4 - bit];
    }
    return fast;
}

// Unit stage on in-block index bit log2(S), both rows at once:
// lo' = lo + b hi, hi' = c lo + hi.
template <int S>
__device__ __forceinline__ void unit_stage(float2 (&p)[32], float b, float c)
{
    const float2 B = make_float2(b, b), C = make_float2(c, c);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        if (i & S) continue;
        const float2 lo = p[i], hi = p[i + S];
        p[i] = __ffma2_rn(B, hi, lo);
        p[i + S] = __ffma2_rn(C, lo, hi);
    }
}

// Direct stage lo' = g00 lo + g01 hi, hi' = g10 lo + g11 hi (variant 2's
// direct_stage2 operation order).
template <int S>
__device__ __forceinline__ void direct_stage(float2 (&p)[32], float4 g)
{
    const float2 F00 = make_float2(g.x, g.x), F01 = make_float2(g.y, g.y);
    const float2 F10 = make_float2(g.z, g.z), F11 = make_float2(g.w, g.w);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        if (i & S) continue;
        const float2 lo = p[i], hi = p[i + S];
        p[i] = __ffma2_rn(F01, hi, __fmul2_rn(F00, lo));
        p[i + S] = __ffma2_rn(F11, hi, __fmul2_rn(F10, lo));
    }
}

// y = D U x for both rows.  D is applied as D*z + (+0), which turns an exact
// zero into +0 whatever the signs (as a cancelling sum does in round-to-
// nearest); bit-identical to kq_fast_apply.
__device__ __forceinline__ void fast_apply(float2 (&p)[32], const Coef &st)
{
    unit_stage<1>(p, st.B[0], st.C[0]);
    unit_stage<2>(p, st.B[1], st.C[1]);
    unit_stage<4>(p, st.B[2], st.C[2]);
    unit_stage<8>(p, st.B[3], st.C[3]);
    unit_stage<16>(p, st.B[4], st.C[4]);
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = __ffma2_rn(p[i], make_float2(st.D[i], st.D[i]), plus_zero2());
}

// The direct form for both rows (columns whose factors the split does not
// admit); bit-identical to kq_direct_apply.
__device__ __forceinline__ void direct_apply(float2 (&p)[32], const float4 (&g)[5])
{
    direct_stage<1>(p, g[4]);
    direct_stage<2>(p, g[3]);
    direct_stage<4>(p, g[2]);
    direct_stage<8>(p, g[1]);
    direct_stage<16>(p, g[0]);
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = __fadd2_rn(p[i], plus_zero2());
}

// Both rows' raw 64-byte blocks -> the pair layout p[i] = (row 0 x_i, row 1 x_i).
__device__ __forceinline__ void unpack_rows(const uint4 (&r0)[4], const uint4 (&r1)[4], float2 (&p)[32])
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t a[4] = {r0[q].x, r0[q].y, r0[q].z, r0[q].w};
        const uint32_t b[4] = {r1[q].x, r1[q].y, r1[q].z, r1[q].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            p[8 * q + 2 * w] = make_float2(bf16_lo(a[w]), bf16_lo(b[w]));
            p[8 * q + 2 * w + 1] = make_float2(bf16_hi(a[w]), bf16_hi(b[w]));
        }
    }
}

// Block amaxes of both rows (NaN-propagating).
__device__ __forceinline__ void amax_rows(const float2 (&p)[32], float &a0, float &a1)
{
    a0 = amax32<true>([&](int i) { return p[i].x; });
    a1 = amax32<true>([&](int i) { return p[i].y; });
}

// MXFP4 of both rows from their amaxes (E8M0 bytes, exact 2^-e scaling,
// E2M1, packing with element 0 in the low nibble of byte 0).
__device__ __forceinline__ void finish_rows(float2 (&p)[32], float a0, float a1, uint4 &c0, uint4 &c1,
                                            uint32_t &s0, uint32_t &s1)
{
    s0 = e8m0_byte(a0);
    s1 = e8m0_byte(a1);
    const float2 ss = make_float2(inv_scale(s0), inv_scale(s1));
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = __fmul2_rn(p[i], ss);
    c0.x = cvt_e2m1x8(p[0].x, p[1].x, p[2].x, p[3].x, p[4].x, p[5].x, p[6].x, p[7].x);
    c0.y = cvt_e2m1x8(p[8].x, p[9].x, p[10].x, p[11].x, p[12].x, p[13].x, p[14].x, p[15].x);
    c0.z = cvt_e2m1x8(p[16].x, p[17].x, p[18].x, p[19].x, p[20].x, p[21].x, p[22].x, p[23].x);
    c0.w = cvt_e2m1x8(p[24].x, p[25].x, p[26].x, p[27].x, p[28].x, p[29].x, p[30].x, p[31].x);
    c1.x = cvt_e2m1x8(p[0].y, p[1].y, p[2].y, p[3].y, p[4].y, p[5].y, p[6].y, p[7].y);
    c1.y = cvt_e2m1x8(p[8].y, p[9].y, p[10].y, p[11].y, p[12].y, p[13].y, p[14].y, p[15].y);
    c1.z = cvt_e2m1x8(p[16].y, p[17].y, p[18].y, p[19].y, p[20].y, p[21].y, p[22].y, p[23].y);
    c1.w = cvt_e2m1x8(p[24].y, p[25].y, p[26].y, p[27].y, p[28].y, p[29].y, p[30].y, p[31].y);
}

constexpr float kFltMax = 3.40282347e38f;

template <int P>
__global__ void __launch_bounds__(Cfg<P>::kThreads, 1)
kq_ring_kernel(const __grid_constant__ CUtensorMap act_map, const uint4 *__restrict__ act,
               const float *__restrict__ factors, int shared, uint4 *__restrict__ codes,
               uint8_t *__restrict__ scales, int64_t nblocks, int nb, long long budget)
{
    pdl_wait();
    using C = Cfg<P>;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(base + size_t(C::kStages) * C::kStageBytes);
    uint64_t *empty = full + C::kStages;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], P / 32);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const int64_t nchunks = (nblocks + P - 1) / P;
    const int64_t G = gridDim.x;

    if (threadIdx.x >= P) {
        // ---------------- producer (one thread): chunk k of this CTA into stage k % kStages
        if (threadIdx.x != P) return;
        int k = 0, filled = 0;
        for (int64_t c = blockIdx.x; c < nchunks; c += G, ++k) {
            const int s = k % C::kStages;
            if (k >= C::kStages && !mbar_wait(&empty[s], ((k / C::kStages) - 1) & 1, budget)) {
                atomicAdd(&g_wait_timeouts, 1);
                break;
            }
            mbar_expect_tx(&full[s], C::kStageBytes);
#pragma unroll
            for (int b = 0; b < C::kBoxes; ++b)
                tma_load_rows(base + size_t(s) * C::kStageBytes + size_t(b) * C::kBoxRows * 64, &act_map,
                              int32_t(c * P + b * C::kBoxRows), &full[s]);
            filled = k + 1;
        }
        // every issued copy has landed before this thread (and so the CTA) exits
        for (int kk = (filled > C::kStages ? filled - C::kStages : 0); kk < filled; ++kk)
            if (!mbar_wait(&full[kk % C::kStages], (kk / C::kStages) & 1, budget)) {
                atomicAdd(&g_wait_timeouts, 1);
                break;
            }
        return;
    }

    // ---------------- consumers: thread t owns row t of every stage
    const int t = threadIdx.x;
    const int lane = t & 31;
    const int j = int((int64_t(blockIdx.x) * P + t) % nb);
    Coef st;
    bool fast;
    {
        float4 g[5];
        load_factors(reinterpret_cast<const float4 *>(factors), shared, j, g);
        fast = coef_setup(g, st);
    }
    const uint32_t row_off = uint32_t(t) * 64;
    const int sw = (t >> 1) & 3;

    bool overflow = false;
    int k = 0;
    for (int64_t c0 = blockIdx.x; c0 < nchunks; c0 += 2 * G, k += 2) {
        const int64_t c1 = c0 + G;
        const bool two = c1 < nchunks;                      // uniform over the CTA
        const int s0 = k % C::kStages, s1 = s0 + 1;
        const uint32_t par = (k / C::kStages) & 1;          // stages s0, s1 are on the same use
        bool ready = mbar_wait(&full[s0], par, budget);
        if (two) ready = ready && mbar_wait(&full[s1], par, budget);
        if (!__all_sync(0xffffffffu, ready)) {
            if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
            return;
        }
        uint4 r0[4], r1[4];
        const uint8_t *row0 = base + size_t(s0) * C::kStageBytes + row_off;
        const uint8_t *row1 = base + size_t(two ? s1 : s0) * C::kStageBytes + row_off;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            r0[q] = *reinterpret_cast<const uint4 *>(row0 + 16 * (q ^ sw));
            r1[q] = *reinterpret_cast<const uint4 *>(row1 + 16 * (q ^ sw));
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&empty[s0]);
            if (two) mbar_arrive(&empty[s1]);
        }
        const int64_t g0 = c0 * P + t, g1 = c1 * P + t;
        float2 p[32];
        unpack_rows(r0, r1, p);
        if (fast) {
            fast_apply(p, st);
        } else {
            // a column the split does not admit: its raw factors are re-read
            // (L1) rather than kept live beside the unit-diagonal ones
            float4 g[5];
            load_factors(reinterpret_cast<const float4 *>(factors), shared, j, g);
            direct_apply(p, g);
        }
        float a0, a1;
        amax_rows(p, a0, a1);
        uint4 w0, w1;
        uint32_t b0, b1;
        finish_rows(p, a0, a1, w0, w1, b0, b1);
        // a block that is not finite: recomputed in the direct form (or 0xFF)
        // a non-finite block: 0xFF and zero codes now; a unit-diagonal one
        // is rewritten by the pass after the loop (kq_redo_overflow)
        if (!(a0 <= kFltMax)) {
            w0 = make_uint4(0u, 0u, 0u, 0u);
            b0 = 0xFFu;
            overflow |= fast;
        }
        if (!(a1 <= kFltMax)) {
            w1 = make_uint4(0u, 0u, 0u, 0u);
            b1 = 0xFFu;
            overflow |= fast;
        }
        if (g0 < nblocks) {
            codes[g0] = w0;
            scales[g0] = uint8_t(b0);
        }
        if (two && g1 < nblocks) {
            codes[g1] = w1;
            scales[g1] = uint8_t(b1);
        }
    }
    // the thread's blocks are g = (blockIdx.x + i G) P + t: stride G P
    if (overflow)
        kq_redo_overflow<KqOut::kCodes, false, false>(act, factors, shared, int64_t(blockIdx.x) * P + t, G * P,
                                                      nblocks, nb, codes, scales, nullptr);
}

}  // namespace ring
