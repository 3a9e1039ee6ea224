// kq_mma.cuh -- KroQuant quantizer with the block transform on the tcgen05
// tensor cores (variant 4).  Included by kroquant.cu; uses its helpers
// (mbarriers, TMA, the MXFP4 epilogue pieces).
//
// Per 32-column block j, Y_j = X_j K_j^T is a [rows x 32] x [32 x 32] product
// (K_j = G1 (x) ... (x) G5 expanded in fp32).  The product must keep fp32
// accuracy (the quantizer's fp32 transform), so K_j is split into three bf16
// parts K_hi + K_mid + K_lo (8 + 8 + 8 significand bits, the rest below fp32
// rounding); X is bf16 already, so each of the three products is exact in the
// fp32 accumulator and Y_j = X_j K_hi^T + X_j K_mid^T + X_j K_lo^T.
//
// The three splits of a block are stacked along N (rows 0-31, 32-63 and
// 64-95 of one K-major B matrix), so one M128 N96 K16 MMA per k-step computes
// all three partial products of a block from one read of its A slice; the
// epilogue adds them in fp32 as (hi + mid) + lo.
//
// A CTA owns one SM (1 CTA/SM, persistent) and walks a contiguous range of
// tiles in group-major order: a tile is 128 rows x kNC = 2 block columns; the
// tiles of one column group share the B operands.
//   warp 0      producer: the TMA load of each A tile (one {64 cols x 128
//               rows} box, 128-byte swizzle) into an 8-stage ring
//   warp 1      allocates the tensor memory; one thread issues the MMAs:
//               2 k-steps x kNC block columns of M128 N96 K16 per tile into
//               accumulator k % 2 (a 128-column slot per block column, 96
//               columns used)
//   warps 2-9   epilogue, two groups of four warps (one per TMEM lane quarter)
//               taking alternate tiles, so each group owns one accumulator:
//               a warp reads its 32 rows' 3 x 32 partial values of both block
//               columns, sums them, releases the accumulator, and quantizes
//               (amax, E8M0 byte, exact 2^-e scaling by a packed FFMA with +0,
//               so exact zeros come out +0 as in the other variants, E2M1).
//               It writes its 32 x 32 bytes of codes with its own TMA store
//               (through a 1 KB staging buffer) and each row's two scale bytes
//               with one 2-byte store.  No barrier joins the epilogue warps.
//   warps 10-13 B builders: at each column-group change they build the group's
//               B set (K_j split into 3 bf16 matrices, K-major, 64-byte
//               swizzle), two of its eight parts per warp, into the B buffer
//               the MMAs released, one set ahead of the MMAs.
// Every mbarrier wait is bounded (g_wait_timeouts); the tensor memory is
// freed on every path.

namespace mma {

constexpr int kNC = 2;                                   // block columns per tile
constexpr int kRows = 128;                               // tile rows (MMA M)
constexpr int kAStages = 8;
constexpr int kABoxBytes = kRows * 128;                  // {64 cols x 128 rows} bf16 = 16 KB
constexpr int kAStageBytes = kABoxBytes;                 // kNC = 2 block columns: one box
constexpr int kBMatBytes = 32 * 64;                      // one 32 x 32 bf16 matrix: 2 KB
constexpr int kBSetBytes = kNC * 3 * kBMatBytes;         // 12 KB
constexpr int kMmaN = 96;                                // the three splits of a block
constexpr int kAccCols = 128;                            // accumulator slot per block column (96 used)
constexpr int kTmemCols = 2 * kNC * kAccCols;            // two accumulators: 512 columns
constexpr int kEpiWarps = 8;                             // two groups of 4 lane quarters
constexpr int kBuildWarps = 4;                           // B builders, two of the 8 parts of a set each
constexpr int kThreads = 64 + 32 * (kEpiWarps + kBuildWarps);   // 448
constexpr int kStoreRows = 32;                           // codes store box: a warp's rows x kNC * 16 bytes
constexpr int kWarpOutBytes = kStoreRows * kNC * 16;     // 1 KB of codes per warp and tile
constexpr size_t kSmemA = size_t(kAStages) * kAStageBytes;
constexpr size_t kSmemB = 2 * size_t(kBSetBytes);
constexpr size_t kSmemOut = size_t(kEpiWarps) * kWarpOutBytes;
constexpr int kNumBars = 2 * kAStages + 8;               // A ring, accumulators, B sets
constexpr size_t kSmemBars = kNumBars * sizeof(uint64_t) + 16;
constexpr size_t kSmem = kSmemA + kSmemB + kSmemOut + kSmemBars + 1024;
static_assert(kNC == 2, "one A box per tile; a row's two scale bytes in one store");
static_assert(kTmemCols <= 512, "tensor memory columns");
static_assert(kSmemB % 1024 == 0 && kSmemA % 1024 == 0, "operand buffers keep the swizzle alignment");
static_assert(kWarpOutBytes % 128 == 0, "TMA store sources stay 128-byte aligned");

// Instruction descriptor (kind::f16): D fp32 (bits 4-5 = 1), A bf16 (bits 7-9
// = 1), B bf16 (bits 10-12 = 1), A and B K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kMmaN >> 3) << 17) |
                            (uint32_t(kRows >> 4) << 24);

// Shared-memory matrix descriptor: start address >> 4 (bits 0-13), leading
// byte offset >> 4 (bits 16-29; unused by swizzled K-major layouts, 1),
// stride byte offset >> 4 (bits 32-45: the distance between 8-row groups),
// version 1 (bits 46-47), base offset 0, layout type in bits 61-63
// (2 = 128-byte swizzle, 4 = 64-byte swizzle).
constexpr uint64_t kLayoutSw128 = 2, kLayoutSw64 = 4;

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t sbo_bytes, uint64_t layout)
{
    return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32) |
           (uint64_t(1) << 46) | (layout << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
                 "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
                 : "memory");
}

// Arrive (once) on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective),
// without the wait: the caller issues several loads and then one
// tcgen05.wait::ld before reading any of them.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int32_t x, int32_t y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half), .y = hi
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Part `part` = 4 jj + c of the B operands of column group g (warp-
// collective; lane n writes row n): chunk c (columns l = 8c .. 8c+7) of row n
// of the three split matrices of block column jj (j = g*kNC + jj).  Matrix
// (jj, s) holds part s of K_j as 32 rows n x 32 columns l (K-major,
// B[n][l] = K_j[n][l], since Y = X K^T), in the 64-byte swizzle layout: row n
// at n*64, its 16-byte chunk c at chunk c ^ ((n >> 1) & 3).  The three
// matrices of a block column are consecutive, so they form one 96-row
// matrix in the same layout.
__device__ void build_b_part(uint8_t *dst, const float4 *__restrict__ factors, int shared, int g, int nb, int lane,
                             int part)
{
    const int jj = part >> 2, c = part & 3;
    const int n = lane;
    const int sw = (n >> 1) & 3;
    const int j = g * kNC + jj;
    float r[5][2];
    if (j < nb) {
        const float4 *fp = factors + (shared ? 0 : int64_t(j) * 5);
#pragma unroll
        for (int k = 0; k < 5; ++k) {
            const float4 f = __ldg(fp + k);            // [g00, g01, g10, g11] of G_(k+1)
            const int bn = (n >> (4 - k)) & 1;          // G_(k+1) acts on index bit 4-k
            r[k][0] = bn ? f.z : f.x;
            r[k][1] = bn ? f.w : f.y;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 5; ++k) r[k][0] = r[k][1] = 0.0f;
    }
    float part_v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int l = 8 * c + e;
        const float a0 = ((l >> 4) & 1) ? r[0][1] : r[0][0];
        const float a1 = ((l >> 3) & 1) ? r[1][1] : r[1][0];
        const float a2 = ((l >> 2) & 1) ? r[2][1] : r[2][0];
        const float a3 = ((l >> 1) & 1) ? r[3][1] : r[3][0];
        const float a4 = (l & 1) ? r[4][1] : r[4][0];
        part_v[e] = a0 * a1 * a2 * a3 * a4;
    }
#pragma unroll
    for (int sp = 0; sp < 3; ++sp) {
        // part sp of the split: round to bf16, carry the exact remainder on
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const __nv_bfloat16 ha = __float2bfloat16_rn(part_v[e]), hb = __float2bfloat16_rn(part_v[e + 1]);
            part_v[e] -= __bfloat162float(ha);
            part_v[e + 1] -= __bfloat162float(hb);
            w[e / 2] = uint32_t(__bfloat16_as_ushort(ha)) | (uint32_t(__bfloat16_as_ushort(hb)) << 16);
        }
        *reinterpret_cast<uint4 *>(dst + (jj * 3 + sp) * kBMatBytes + n * 64 + 16 * (c ^ sw)) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int32_t x, int32_t y, const void *src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_addr(src))
                 : "memory");
}

// Sum of the three partial products of one block column at TMEM address
// `tcol` (this warp's lane quarter): (hi + mid) + lo in fp32.
__device__ __forceinline__ void load_block_sum(uint32_t tcol, float (&y)[32])
{
    float u[32], w[32];
    tmem_ld32_nowait(tcol, y);
    tmem_ld32_nowait(tcol + 32, u);
    tmem_ld32_nowait(tcol + 64, w);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 s = __fadd2_rn(__fadd2_rn(make_float2(y[2 * i], y[2 * i + 1]), make_float2(u[2 * i], u[2 * i + 1])),
                                    make_float2(w[2 * i], w[2 * i + 1]));
        y[2 * i] = s.x;
        y[2 * i + 1] = s.y;
    }
}

// MXFP4 of one block's 32 transformed values (amax, E8M0 byte, exact 2^-e
// scaling by a packed FFMA with +0, E2M1); a block that is not finite gets
// the E8M0 NaN byte 0xFF and zero codes.
__device__ __forceinline__ void quantize_block32(float (&v)[32], uint4 &cw, uint32_t &sb)
{
    const float amax = amax32<true>([&](int i) { return v[i]; });
    if (!(amax <= 3.40282347e38f)) {
        cw = make_uint4(0u, 0u, 0u, 0u);
        sb = 0xFFu;
        return;
    }
    sb = e8m0_byte(amax);
    const float sc = inv_scale(sb);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 pr = __ffma2_rn(make_float2(v[2 * i], v[2 * i + 1]), make_float2(sc, sc), plus_zero2());
        v[2 * i] = pr.x;
        v[2 * i + 1] = pr.y;
    }
    cw.x = cvt_e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
    cw.y = cvt_e2m1x8(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
    cw.z = cvt_e2m1x8(v[16], v[17], v[18], v[19], v[20], v[21], v[22], v[23]);
    cw.w = cvt_e2m1x8(v[24], v[25], v[26], v[27], v[28], v[29], v[30], v[31]);
}

template <KqOut OUT>
__global__ void __launch_bounds__(kThreads, 1)
kq_mma_kernel(const __grid_constant__ CUtensorMap act_map, const __grid_constant__ CUtensorMap codes_map,
              const float4 *__restrict__ factors, int shared, uint8_t *__restrict__ scales,
              float4 *__restrict__ y_out, int64_t M, int nb, long long budget)
{
    pdl_wait();
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = base + kSmemA;
    uint8_t *sOut = sB + kSmemB;                               // [kEpiWarps] x a warp's codes (32 rows x 32 bytes)
    uint64_t *bars = reinterpret_cast<uint64_t *>(sOut + kSmemOut);
    uint64_t *full_a = bars;                  // [kAStages] A tile landed (TMA tx)
    uint64_t *empty_a = bars + kAStages;      // [kAStages] MMAs reading the stage done (commit)
    uint64_t *tfull = bars + 2 * kAStages;    // [2] accumulator ready (commit)
    uint64_t *tempty = tfull + 2;             // [2] accumulator read by its epilogue group
    uint64_t *bfull = tfull + 4;              // [2] B set built (the builder warps)
    uint64_t *bempty = tfull + 6;             // [2] MMAs reading the B set done (commit)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int64_t RT = (M + kRows - 1) / kRows;
    const int ngroups = (nb + kNC - 1) / kNC;
    const int64_t T = RT * ngroups;
    const int64_t t_begin = int64_t(blockIdx.x) * T / gridDim.x;
    const int64_t t_end = int64_t(blockIdx.x + 1) * T / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&empty_a[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
            mbar_init(&bfull[b], kBuildWarps);
            mbar_init(&bempty[b], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- producer: A tiles (one thread)
        if (lane == 0) {
            int filled = 0;
            int k = 0;
            for (int64_t t = t_begin; t < t_end; ++t, ++k) {
                const int g = int(t / RT);
                const int64_t rt = t % RT;
                const int s = k % kAStages;
                if (k >= kAStages && !mbar_wait(&empty_a[s], ((k / kAStages) - 1) & 1, budget)) {
                    atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
                mbar_expect_tx(&full_a[s], kAStageBytes);
                tma_load_2d(sA + size_t(s) * kAStageBytes, &act_map, g * kNC * 32, int32_t(rt * kRows), &full_a[s]);
                filled = k + 1;
            }
            // drain: the copies issued have landed before the CTA may exit
            for (int kk = (filled > kAStages ? filled - kAStages : 0); kk < filled; ++kk)
                if (!mbar_wait(&full_a[kk % kAStages], (kk / kAStages) & 1, budget)) {
                    atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            int last_g = -1, bcount = -1, k = 0, issued = 0;
            for (int64_t t = t_begin; t < t_end; ++t, ++k) {
                const int g = int(t / RT);
                if (g != last_g) {
                    if (bcount >= 0) umma_commit(&bempty[bcount & 1]);
                    ++bcount;
                    if (!mbar_wait(&bfull[bcount & 1], (bcount >> 1) & 1, budget)) {
                        atomicAdd(&g_wait_timeouts, 1);
                        break;
                    }
                    last_g = g;
                }
                const int s = k % kAStages;
                if (!mbar_wait(&full_a[s], (k / kAStages) & 1, budget)) {
                    atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
                const int tb = k & 1;
                if (k >= 2 && !mbar_wait(&tempty[tb], ((k >> 1) - 1) & 1, budget)) {
                    atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = smem_addr(sA + size_t(s) * kAStageBytes);
                const uint32_t b0 = smem_addr(sB + (bcount & 1) * kBSetBytes);
                // Block column innermost: the two MMAs that accumulate into
                // one slot are kNC issues apart.  Block column jj's 32 A
                // columns are bytes 64 jj .. 64 jj + 63 of the 128-byte rows;
                // its B matrix is the 96 stacked split rows.
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                    for (int jj = 0; jj < kNC; ++jj) {
                        const uint32_t d = tmem_base + uint32_t(tb * kNC * kAccCols + jj * kAccCols);
                        const uint64_t ad = smem_desc(a0 + jj * 64 + kk * 32, 1024, kLayoutSw128);
                        const uint64_t bd = smem_desc(b0 + jj * 3 * kBMatBytes + kk * 32, 512, kLayoutSw64);
                        umma_bf16(d, ad, bd, kk != 0);
                    }
                }
                umma_commit(&empty_a[s]);
                umma_commit(&tfull[tb]);
                issued = k + 1;
            }
            // every MMA issued has completed before the tensor memory is freed
            if (issued > 0 && !mbar_wait(&tfull[(issued - 1) & 1], ((issued - 1) >> 1) & 1, budget))
                atomicAdd(&g_wait_timeouts, 1);
        }
    } else if (warp < 2 + kEpiWarps) {
        // ---------------- epilogue: group gr takes the tiles k with k % 2 == gr
        // (accumulator gr); warp w reads TMEM lane quarter w % 4 (tile rows
        // 32q .. 32q+31), both block columns
        const int q = warp & 3;
        const int gr = (warp - 2) >> 2;
        uint8_t *stg = sOut + size_t(warp - 2) * kWarpOutBytes;
        int k = 0;
        for (int64_t t = t_begin; t < t_end; ++t, ++k) {
            if ((k & 1) != gr) continue;
            const int use = k >> 1;
            const bool ready = mbar_wait(&tfull[gr], use & 1, budget);
            if (!__all_sync(0xffffffffu, ready)) {   // tcgen05.ld below is warp-collective
                if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                break;
            }
            tc_fence_after();
            const int g = int(t / RT);
            const int64_t rt = t % RT;
            const int64_t row0 = rt * kRows + q * 32;
            const int64_t row = row0 + lane;
            const int j0 = g * kNC;
            const uint32_t tcol = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(gr * kNC * kAccCols);
            float y[32];
            if constexpr (OUT == KqOut::kF32) {
#pragma unroll 1
                for (int jj = 0; jj < kNC; ++jj) {
                    load_block_sum(tcol + jj * kAccCols, y);
                    if (row < M && j0 + jj < nb) {
                        // the fp32 transform itself (+0: exact zeros come out +0)
                        float4 *yo = y_out + (row * nb + j0 + jj) * 8;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            yo[i] = make_float4(y[4 * i] + 0.0f, y[4 * i + 1] + 0.0f, y[4 * i + 2] + 0.0f,
                                                y[4 * i + 3] + 0.0f);
                    }
                }
                // both block columns have been read: hand the accumulator back
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[gr]);
            } else {
                uint4 cw0, cw1;
                uint32_t sb0, sb1;
                load_block_sum(tcol, y);
                quantize_block32(y, cw0, sb0);
                load_block_sum(tcol + kAccCols, y);
                // both block columns have been read: hand the accumulator back
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[gr]);
                quantize_block32(y, cw1, sb1);
                // this warp's codes: 32 rows x 32 bytes through its staging
                // buffer (the previous store has finished reading it) and one
                // TMA store; rows past M and columns past d/2 are clipped
                if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                __syncwarp();
                *reinterpret_cast<uint4 *>(stg + lane * 32) = cw0;
                *reinterpret_cast<uint4 *>(stg + lane * 32 + 16) = cw1;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0 && row0 < M) {
                    tma_store_2d(&codes_map, j0 * 16, int32_t(row0), stg);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
                // the row's two scale bytes, one 2-byte store where the layout allows it
                if (row < M) {
                    uint8_t *dst = scales + row * nb + j0;
                    if (j0 + 1 < nb && (reinterpret_cast<uintptr_t>(dst) & 1) == 0) {
                        *reinterpret_cast<uint16_t *>(dst) = uint16_t(sb0 | (sb1 << 8));
                    } else {
                        dst[0] = uint8_t(sb0);
                        if (j0 + 1 < nb) dst[1] = uint8_t(sb1);
                    }
                }
            }
        }
        if constexpr (OUT == KqOut::kCodes) {
            if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        }
    } else {
        // ---------------- B builders: warp bw builds parts 2 bw and 2 bw + 1 of
        // each column group's B set, one set ahead of the MMAs where the
        // second buffer is free
        const int bw = warp - 2 - kEpiWarps;
        int last_g = -1, buse = -1;
        for (int64_t t = t_begin; t < t_end; ++t) {
            const int g = int(t / RT);
            if (g == last_g) continue;
            ++buse;
            const int bb = buse & 1;
            // every lane waits (each acquires the release of the old B set);
            // the give-up decision is made warp-uniform
            const bool freed = buse < 2 || mbar_wait(&bempty[bb], ((buse >> 1) - 1) & 1, budget);
            if (!__all_sync(0xffffffffu, freed)) {
                if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                break;
            }
            build_b_part(sB + bb * kBSetBytes, factors, shared, g, nb, lane, 2 * bw);
            build_b_part(sB + bb * kBSetBytes, factors, shared, g, nb, lane, 2 * bw + 1);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&bfull[bb]);
            last_g = g;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace mma
