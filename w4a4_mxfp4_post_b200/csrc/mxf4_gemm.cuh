// mxf4_gemm.cuh -- the W4A4 linear layer that consumes the quantizer's output.
// Included by kroquant.cu; uses its helpers (mbarriers, TMA, descriptors of
// kq_mma.cuh).
//
// D[m][n] = sum_k a[m][k] b[n][k], where a = MXFP4(X T^T) [M x K] is the
// quantized activation and b = MXFP4(W T^-1) [N x K] the quantized folded
// weight ("KroQuant: Kronecker-Structured Block Transforms for Efficient
// Post-Training Quantization of Diffusion Transformers", abstract: W4A4 at
// MXFP4; section 3.2, Eq. (4): the inverse folded into the weights).  Both
// operands are K-major as the quantizers write them (codes [rows][K/2], even
// element in the low nibble), with their E8M0 scales in the scale-factor
// layout (SfPos in kroquant.cu).  D is bf16 or fp32, [M][N] row-major.
//
// One tcgen05 block-scaled MMA (kind::mxf4, block32) is M128 x BN x K64 (BN =
// 256 or 192): the tensor core decodes E2M1 and applies the two E8M0 scales of
// every 32-block, accumulating in fp32 in tensor memory.  The scale bytes reach
// tensor memory by tcgen05.cp from shared memory (one 512-byte unit = 128 rows
// x 4 blocks per copy, 32 lanes x 128 bits replicated to the four lane
// quarters).
//
// Two kernels: the one-SM form below (configurations 1-6, the default up to
// 128 rows) and the SM-pair form (configurations 7 and 8, the default above
// 128 rows), described before mxf4_gemm_pair_kernel.
//
// One-SM form.  A CTA owns one SM (persistent) and walks the 128 x BN output
// tiles t = blockIdx.x, + gridDim.x, ...; a k-chunk is CB bytes of codes per
// row (2 CB elements, one CB-byte swizzle atom; CB / 64 scale units per row
// group), CB, the ring depth ST and BN being compile-time choices (Cfg).
// Every issuing role runs its loop on the whole warp with warp-uniform
// operands, and one elected lane issues.
//   warp 0     producer: per chunk, TMA loads of the A box {CB x 128 rows}
//              and the B box {CB x BN rows} (CB-byte swizzle; rows and bytes
//              past the matrix read as zero) and bulk copies of the chunk's
//              scale units (A: its row group's, B: the tile's two row groups')
//              into an ST-stage ring
//   warp 1     allocates tensor memory; issues the chunk's CB / 32 MMAs (only
//              the K=64 steps below K) once the copier has put the stage's
//              scales in tensor memory, and commits the stage back to the
//              producer; after a tile's last chunk it commits the
//              accumulator.  Where two accumulators fit beside the scale
//              columns (BN = 192) tiles alternate between them.
//   warp 10    the scale copier: copies each landed stage's scale units to
//              that stage's own tensor-memory columns (so a copy never waits
//              on MMAs still reading an older stage) and commits them to the
//              stage's `sf_ready` barrier.  A tcgen05 instruction holds its
//              issuing warp for tens of cycles, so the copies of stage s + 1
//              go out while the MMA warp issues stage s.
//   warps 2-9  epilogue: warp w reads accumulator lanes 32 (w % 4) .. +31 (tile
//              rows) and columns BN/2 ((w - 2) / 4) .. + BN/2 - 1 into
//              registers and hands the accumulator back at once; then, while
//              the MMAs of the next tile run, it stores its segment: with
//              TMA_OUT (bf16) through the warp's 8 KB of shared memory and TMA
//              tensor stores of {64 columns x 32 rows} (128-byte swizzle, BN =
//              256) or {32 x 32} (64-byte swizzle, BN = 192), rows and columns
//              past D clipped; otherwise with 16-byte stores from registers
// Every mbarrier wait is bounded (g_wait_timeouts); every path drains the
// copies in flight, waits for its MMAs and frees the tensor memory.

namespace gemm {

constexpr int kBM = 128;                                  // tile rows (MMA M)
constexpr int kSfUnit = 512;                              // 128 rows x 4 blocks
constexpr int kTmemCols = 512;                            // power of two >= 256 + scale columns
constexpr uint32_t kAccCol = 0;                           // fp32 accumulator(s), then the scale columns
constexpr int kEpiWarps = 8;
constexpr int kCopyWarp = 2 + kEpiWarps;                 // the scale copier (warp 10)
constexpr int kThreads = 96 + 32 * kEpiWarps;             // 352
constexpr int kStageOutBytes = 32 * 128 * 2;              // a warp's 32 rows x 128 bf16 columns
constexpr size_t kSmemMax = 232448;                       // 227 KB per CTA

// Tile configuration: CB codes bytes per row per k-chunk (64 or 128), ST ring
// stages, TMA_OUT = bf16 output through shared memory and TMA stores, BN tile
// columns (256, or 192 where 256-column tiles fill the last wave badly).
// Scale columns per stage and k-unit: A's unit at +0, B's two units at +8 and
// +12 (every tcgen05.cp destination a multiple of 4 columns).  A 192-column
// tile may start in the middle of a 128-row scale unit (odd tiles start at its
// third 32-row group): the MMA then reads B's scales from +10 instead of +8.
template <int CB, int ST, bool TMA_OUT, int BN = 256>
struct Cfg {
    static constexpr int kCB = CB;
    static constexpr int kST = ST;
    static constexpr bool kTmaOut = TMA_OUT;
    static constexpr int kBN = BN;
    static constexpr int kUnits = CB / 64;                // scale units per row group per chunk
    static constexpr int kMmas = CB / 32;                 // K=64 MMAs per chunk
    static constexpr int kABytes = kBM * CB;
    static constexpr int kBBytes = BN * CB;
    static constexpr int kSfaBytes = kUnits * kSfUnit;
    static constexpr int kSfbBytes = 2 * kUnits * kSfUnit;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr uint32_t kSfStageCols = 16 * kUnits;
    static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (1u << 23) |
                                       (uint32_t(kBM >> 4) << 24);
    static constexpr int kEpiCols = BN / 2;               // columns per epilogue warp
    static constexpr uint64_t kLayout = CB == 128 ? mma::kLayoutSw128 : mma::kLayoutSw64;
    static constexpr uint32_t kSbo = 8 * CB;              // 8-row swizzle atom
    static constexpr size_t kRing = size_t(ST) * kStageBytes;
    // Two accumulators where they fit beside the scale columns (192-column
    // tiles: 2 x 192 + scales <= 512): the MMAs of the next tile then start
    // while the epilogue still drains the previous one.
    static constexpr int kAccBufs = (2 * BN + ST * int(16 * (CB / 64)) <= kTmemCols) ? 2 : 1;
    static constexpr uint32_t kSfCol = uint32_t(kAccBufs * BN);   // scale columns: 16 per stage and k-unit
    static constexpr size_t kSmem = kRing + (TMA_OUT ? size_t(kEpiWarps) * kStageOutBytes : 0) + 1024 +
                                    (3 * ST + 6) * sizeof(uint64_t) + 16;
    static_assert(CB == 64 || CB == 128, "chunk bytes");
    static_assert(BN == 256 || BN == 192, "tile columns");
    static_assert(kStageBytes % (8 * CB) == 0, "stages keep the alignment of the swizzle atom");
    static_assert(!TMA_OUT || kRing % 1024 == 0, "the output staging keeps the 1 KB alignment of its swizzle");
    static_assert(kSfCol + ST * kSfStageCols <= kTmemCols, "tensor memory columns");
    static_assert(kSfCol % 4 == 0, "scale columns are 4-aligned");
    static_assert(kSmem <= kSmemMax, "shared memory");
};

// Instruction descriptor (Cfg::kIdesc), block-scaled kinds: b_sf_id bits 4-5,
// A format bits 7-9 and B format bits 10-12 (1 = E2M1 for kind::mxf4),
// K-major A and B (bits 15, 16 = 0), N >> 3 in bits 17-22, scale format bit 23
// (1 = E8M0), M >> 4 in bits 24-28, a_sf_id bits 29-30, bit 31 = 0 (K = 64).
// sf_id selects the byte pair of each 32-bit scale word: the K=64 step j of a
// 128-element unit reads blocks 2j and 2j+1, i.e. bytes 2j, 2j+1 (sf_id 2j).
__device__ __forceinline__ uint32_t idesc(uint32_t base, uint32_t sf_id) { return base | (sf_id << 4) | (sf_id << 29); }

// The MMA and scale-copy warps run their loops with the whole warp, on
// warp-uniform operands, and each tcgen05 instruction below is issued by the
// one lane elect.sync picks: the operands then stay in uniform registers, and
// the issuing thread is not held up moving them there one at a time.
__device__ __forceinline__ void umma_mxf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t id,
                                          uint32_t tmem_sfa, uint32_t tmem_sfb, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                     tmem_d),
                 "l"(adesc), "l"(bdesc), "r"(id), "r"(accumulate), "r"(tmem_sfa), "r"(tmem_sfb)
                 : "memory");
}

// One 512-byte scale unit (shared memory, 32 rows x 16 bytes, no swizzle) to
// 4 tensor-memory columns, replicated to the four 32-lane quarters (whole warp).
__device__ __forceinline__ void tmem_copy_unit(uint32_t taddr, uint32_t saddr)
{
    const uint64_t desc = mma::smem_desc(saddr, 128, 0);
    asm volatile("{\n\t.reg .pred e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr), "l"(desc) : "memory");
}

// Arrive (once) on `bar` when the tcgen05 operations issued so far completed (whole warp).
__device__ __forceinline__ void umma_commit_w(uint64_t *bar)
{
    asm volatile("{\n\t.reg .pred e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

// A bounded wait taken by the whole warp: true only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, long long budget)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, budget));
}

// True in the one lane of the (converged) warp that elect.sync picks.
__device__ __forceinline__ bool elect_one()
{
    uint32_t e;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(e));
    return e != 0;
}

// Plain (untiled) bulk copy global -> shared, completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// 32 fp32 columns of this thread's lane, no wait (the caller waits once).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float *v)
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// One epilogue warp's share of a finished tile: accumulator lanes (rows)
// row0 .. row0 + 31 and EC columns from col0, read from tensor memory at
// taddr.  `release` (lane 0) hands the accumulator back as soon as it is in
// registers; the stores follow: with STAGED (bf16) through the warp's 8 KB of
// shared memory `stg` and TMA tensor stores of {64 columns x 32 rows}
// (128-byte swizzle, EC = 128) or {32 x 32} (64-byte swizzle, EC = 96), rows
// and columns past D clipped; otherwise with 16-byte stores from registers.
//
// SMALL (with STAGED): the warp's staging is two 2 KB buffers used in turn,
// one {32 x 32} box (64-byte swizzle) each; `nbox` counts the boxes this warp
// has staged so far (the buffer of a box is nbox % 2, and before it is
// rewritten the store issued from it two boxes earlier has finished reading
// it).  Every box commits one bulk group, empty where nothing is stored, so
// that "all but the latest group" always covers the buffer's previous store.
template <int EC, bool F32OUT, bool STAGED, bool SMALL = false, class Release>
__device__ __forceinline__ void epilogue_tile(uint32_t taddr, int row0, int col0, int M, int N, void *__restrict__ out,
                                              const CUtensorMap *out_map, uint8_t *stg, Release release,
                                              int *nbox = nullptr)
{
    const int lane = threadIdx.x % 32;
    if constexpr (F32OUT) {
        float v[EC];
#pragma unroll
        for (int i = 0; i < EC / 32; ++i) tmem_ld32_nowait(taddr + 32 * i, v + 32 * i);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        mma::tc_fence_before();
        __syncwarp();
        if (lane == 0) release();
        const int row = row0 + lane;
        if (row < M) {
            float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + int64_t(row) * N + col0);
#pragma unroll
            for (int i = 0; i < EC / 4; ++i)
                if (col0 + 4 * i < N) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    } else {
        // every load in flight at once, one wait, then the accumulator goes
        // back before the packing into bf16 pairs
        uint32_t w[EC / 2];
        {
            float v[EC];
#pragma unroll
            for (int i = 0; i < EC / 32; ++i) tmem_ld32_nowait(taddr + 32 * i, v + 32 * i);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            mma::tc_fence_before();
            __syncwarp();
            if (lane == 0) release();
#pragma unroll
            for (int e = 0; e < EC / 2; ++e) w[e] = mma::pack_bf16x2(v[2 * e], v[2 * e + 1]);
        }
        if constexpr (STAGED && SMALL) {
#pragma unroll
            for (int bx = 0; bx < EC / 32; ++bx) {
                uint8_t *buf = stg + (*nbox & 1) * 2048;
                if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                __syncwarp();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int i = 4 * bx + cc;
                    *reinterpret_cast<uint4 *>(buf + lane * 64 + ((cc ^ ((lane >> 1) & 3)) << 4)) =
                        make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    if (row0 < M && col0 + 32 * bx < N) mma::tma_store_2d(out_map, col0 + 32 * bx, row0, buf);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
                ++*nbox;
            }
        } else if constexpr (STAGED) {
            // the previous tile's stores have finished reading the staging buffer
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();
            if constexpr (EC == 128) {
                // two boxes of 64 columns, 128-byte swizzle: chunk ^ (row % 8)
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int bx = i >> 3, cc = i & 7;
                    *reinterpret_cast<uint4 *>(stg + bx * 4096 + lane * 128 + ((cc ^ (lane & 7)) << 4)) =
                        make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            } else {
                // three boxes of 32 columns, 64-byte swizzle: chunk ^ ((row / 2) % 4)
#pragma unroll
                for (int i = 0; i < 12; ++i) {
                    const int bx = i >> 2, cc = i & 3;
                    *reinterpret_cast<uint4 *>(stg + bx * 2048 + lane * 64 + ((cc ^ ((lane >> 1) & 3)) << 4)) =
                        make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            // boxes that start past D are not issued; the rest is clipped
            if (lane == 0 && row0 < M && col0 < N) {
                constexpr int BW = EC == 128 ? 64 : 32;            // box width (columns)
#pragma unroll
                for (int bx = 0; bx < EC / BW; ++bx)
                    if (col0 + BW * bx < N) mma::tma_store_2d(out_map, col0 + BW * bx, row0, stg + bx * BW * 64);
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
        } else {
            const int row = row0 + lane;
            if (row < M) {
                uint4 *o = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + int64_t(row) * N + col0);
#pragma unroll
                for (int i = 0; i < EC / 8; ++i)
                    if (col0 + 8 * i < N) o[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
    }
}

template <class C, bool F32OUT>
__global__ void __launch_bounds__(kThreads, 1)
mxf4_gemm_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap b_map,
                 const __grid_constant__ CUtensorMap out_map, const uint8_t *__restrict__ a_sf,
                 const uint8_t *__restrict__ b_sf, void *__restrict__ out, int M, int N, int K, long long budget)
{
    pdl_wait();
    constexpr int ST = C::kST;
    constexpr int kBN = C::kBN;
    constexpr bool kStaged = C::kTmaOut && !F32OUT;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t *stage_out = base + C::kRing;                // [kEpiWarps] x 8 KB output staging (TMA_OUT)
    uint64_t *bars = reinterpret_cast<uint64_t *>(stage_out + (C::kTmaOut ? size_t(kEpiWarps) * kStageOutBytes : 0));
    uint64_t *full = bars;                    // [ST] stage landed (TMA / bulk tx)
    uint64_t *empty = bars + ST;              // [ST] MMAs reading the stage done (commit)
    uint64_t *sf_ready = bars + 2 * ST;       // [ST] the stage's scale units are in tensor memory (commit)
    constexpr int NA = C::kAccBufs;
    uint64_t *acc_full = bars + 3 * ST;       // [2] accumulator b holds a finished tile (commit)
    uint64_t *acc_empty = acc_full + 2;       // [2] accumulator b read by the 8 epilogue warps
    uint64_t *done = acc_full + 4;            // every MMA of this CTA completed (final commit)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 6);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int MT = (M + kBM - 1) / kBM;
    const int NT = (N + kBN - 1) / kBN;
    const int tiles = MT * NT;
    const int KC = (K + 2 * C::kCB - 1) / (2 * C::kCB);   // k-chunks
    const int Ka = (K + 127) / 128;                       // scale units per 128-row group
    const int KS = (K + 63) / 64;                         // MMA K steps
    const int NRa = (N + 127) / 128;                      // B row groups with scale units

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_ready[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps);
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    mma::tc_fence_before();
    __syncthreads();
    mma::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        {
            // ---------------- producer (the whole warp; one elected lane issues)
            int k = 0, filled = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int mt = t / NT, nt = t % NT;
                const int g0 = nt * kBN / 128;                // first B row group of the tile
                const bool b_hi = g0 + 1 < NRa;               // its second row group exists
                for (int c = 0; c < KC; ++c, ++k) {
                    const int s = k % ST;
                    if (k >= ST && !warp_wait(&empty[s], ((k / ST) - 1) & 1, budget)) {
                        if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                        ok = false;
                        break;
                    }
                    uint8_t *st = base + size_t(s) * C::kStageBytes;
                    uint8_t *sfa = st + C::kABytes + C::kBBytes;
                    uint8_t *sfb = sfa + C::kSfaBytes;
                    const int u0 = c * C::kUnits;
                    const int nu = Ka - u0 < C::kUnits ? Ka - u0 : C::kUnits;   // units of this chunk, >= 1
                    const uint32_t sfbytes = uint32_t(nu) * kSfUnit;
                    if (elect_one()) {
                        mbar_expect_tx(&full[s], uint32_t(C::kABytes + C::kBBytes) + sfbytes * (b_hi ? 3u : 2u));
                        mma::tma_load_2d(st, &a_map, c * C::kCB, mt * kBM, &full[s]);
                        mma::tma_load_2d(st + C::kABytes, &b_map, c * C::kCB, nt * kBN, &full[s]);
                        bulk_load(sfa, a_sf + (int64_t(mt) * Ka + u0) * kSfUnit, sfbytes, &full[s]);
                        bulk_load(sfb, b_sf + (int64_t(g0) * Ka + u0) * kSfUnit, sfbytes, &full[s]);
                        if (b_hi)
                            bulk_load(sfb + C::kUnits * kSfUnit, b_sf + (int64_t(g0 + 1) * Ka + u0) * kSfUnit,
                                      sfbytes, &full[s]);
                    }
                    __syncwarp();
                    filled = k + 1;
                }
            }
            // drain: the copies issued have landed before the CTA may exit
            for (int kk = (filled > ST ? filled - ST : 0); kk < filled; ++kk)
                if (!warp_wait(&full[kk % ST], (kk / ST) & 1, budget)) {
                    if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
        }
    } else if (warp == 1) {
        // ---------------- MMAs (the whole warp; one elected lane issues)
        {
            int k = 0, it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++it) {
                // a tile starting mid-unit (192-column tiles): the MMA reads B's
                // scales off = 0 or 2 columns (32-row groups) into the first unit
                const uint32_t off = uint32_t(((t % NT) * kBN % 128) / 32);
                const int ab = it % NA;               // accumulator of this tile
                if (it >= NA && !warp_wait(&acc_empty[ab], ((it / NA) - 1) & 1, budget)) {
                    if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
                mma::tc_fence_after();
                for (int c = 0; c < KC; ++c, ++k) {
                    const int s = k % ST;
                    // the stage landed and the copier has put its scale units in tensor memory
                    if (!warp_wait(&full[s], (k / ST) & 1, budget) || !warp_wait(&sf_ready[s], (k / ST) & 1, budget)) {
                        if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                        ok = false;
                        break;
                    }
                    mma::tc_fence_after();
                    const uint32_t a0 = smem_addr(base + size_t(s) * C::kStageBytes);
                    const uint32_t b0 = a0 + C::kABytes;
                    const uint32_t tsf = tmem_base + C::kSfCol + uint32_t(s) * C::kSfStageCols;   // + 16 u
#pragma unroll
                    for (int j = 0; j < C::kMmas; ++j) {
                        if (c * C::kMmas + j >= KS) break;
                        const uint32_t sf_id = 2 * (j & 1);
                        const uint32_t u = j >> 1;
                        const uint64_t ad = mma::smem_desc(a0 + j * 32, C::kSbo, C::kLayout);
                        const uint64_t bd = mma::smem_desc(b0 + j * 32, C::kSbo, C::kLayout);
                        umma_mxf4(tmem_base + kAccCol + uint32_t(ab * kBN), ad, bd, idesc(C::kIdesc, sf_id),
                                  (tsf + 16 * u) | (sf_id << 30),
                                  (tsf + 16 * u + 8 + off) | (sf_id << 30), (c | j) != 0);
                    }
                    umma_commit_w(&empty[s]);
                }
                if (!ok) break;
                umma_commit_w(&acc_full[ab]);
            }
            // every MMA issued has completed before the tensor memory is freed
            umma_commit_w(done);
            if (!warp_wait(done, 0, budget) && lane == 0) atomicAdd(&g_wait_timeouts, 1);
        }
    } else if (warp == kCopyWarp) {
        {
            // ---------------- scale copies (the whole warp): each stage's units to
            // that stage's own tensor-memory columns, so a copy never waits on
            // MMAs still reading an older stage, and the MMA thread only issues
            // MMAs.  Units past K or of a missing B row group are stale data:
            // they reach only K steps not issued or output columns >= N.
            int k = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                for (int c = 0; c < KC; ++c, ++k) {
                    const int s = k % ST;
                    if (!warp_wait(&full[s], (k / ST) & 1, budget)) {
                        if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                        ok = false;
                        break;
                    }
                    mma::tc_fence_after();
                    const uint32_t sfa = smem_addr(base + size_t(s) * C::kStageBytes) + C::kABytes + C::kBBytes;
                    const uint32_t sfb = sfa + C::kSfaBytes;
                    const uint32_t tsf = tmem_base + C::kSfCol + uint32_t(s) * C::kSfStageCols;
#pragma unroll
                    for (int u = 0; u < C::kUnits; ++u) {
                        tmem_copy_unit(tsf + 16 * u, sfa + u * kSfUnit);
                        tmem_copy_unit(tsf + 16 * u + 8, sfb + u * kSfUnit);
                        tmem_copy_unit(tsf + 16 * u + 12, sfb + (C::kUnits + u) * kSfUnit);
                    }
                    umma_commit_w(&sf_ready[s]);
                    issued = k + 1;
                }
            }
            // the copies issued have completed before the tensor memory is freed
            if (issued > 0 && !warp_wait(&sf_ready[(issued - 1) % ST], ((issued - 1) / ST) & 1, budget) && lane == 0)
                atomicAdd(&g_wait_timeouts, 1);
        }
    } else {
        // ---------------- epilogue
        const int q = warp & 3;                   // lane quarter this warp may read
        const int h = (warp - 2) >> 2;            // column half of the tile
        int it = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
            const int mt = t / NT, nt = t % NT;
            const int ab = it % NA;
            const bool ready = mbar_wait(&acc_full[ab], (it / NA) & 1, budget);
            if (!__all_sync(0xffffffffu, ready)) {   // tcgen05.ld below is warp-collective
                if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                break;
            }
            mma::tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + kAccCol + uint32_t(ab * kBN + h * C::kEpiCols);
            epilogue_tile<C::kEpiCols, F32OUT, kStaged>(taddr, mt * kBM + q * 32, nt * kBN + h * C::kEpiCols, M, N, out,
                                                        &out_map, stage_out + size_t(warp - 2) * kStageOutBytes,
                                                        [&] { mbar_arrive(&acc_empty[ab]); });
        }
        if constexpr (kStaged) {
            if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        }
    }

    mma::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        mma::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// The SM-pair form (cta_group::2).  A cluster of two CTAs on two SMs computes
// a 256 x BN output tile; one M256 x BN x K64 block-scaled MMA per K step is
// issued by the cluster's rank-0 CTA (the leader) and runs on both SMs.  Each
// CTA stages, per 256-element k-chunk, its own 128 rows of A, its half (BN/2
// rows) of B, the scale units of its A row group and those of both B row
// groups the tile touches (the tensor core of each SM reads the B scales of
// all BN columns from its own tensor memory).  An SM so moves 128 + BN/2
// operand rows per 128 x BN outputs where the one-SM form moves 128 + BN.
//   warp 0     producer (both CTAs): TMA loads in the .cta_group::2 form,
//              completing on the LEADER's `full` barrier of the stage, which
//              the leader arms with both CTAs' bytes; the operands as in the
//              one-SM form, the scale units as 3-D boxes {256 B x 4 x 1 or 2
//              row groups} (units past K or row groups past the matrix read
//              as zero)
//   warp 1     allocates the pair's tensor memory (.cta_group::2, both CTAs);
//              in the leader the warp (one elected lane) issues the MMAs and commits each stage
//              to the `empty` barrier of both CTAs and each finished tile to
//              the `acc_full` barrier of both
//   warp 10    in the leader, the scale copier: each stage's scale units into
//              both SMs' tensor memory (tcgen05.cp .cta_group::2: each CTA's
//              shared memory to its own tensor memory), committed to the
//              leader's `sf_ready` barrier of the stage
//   warps 2-9  epilogue (both CTAs) as in the one-SM form, on the CTA's own
//              128 accumulator lanes; the accumulator is handed back by an
//              arrival on the LEADER's `acc_empty` (16 arrivals, 8 per CTA);
//              bf16 stores go out as {32 x 32} TMA boxes through two 2 KB
//              buffers per warp, which leaves the shared memory to a deeper
//              ring (the loads' round trip, not their bandwidth, limits it)
// No load reads another GPU's memory and none is multicast.  Every mbarrier
// wait is bounded; a cluster barrier that every path reaches precedes the
// release of the tensor memory.
template <int BN, int ST>
struct PairCfg {
    static constexpr int kCB = 128;                       // codes bytes per row per k-chunk
    static constexpr int kST = ST;
    static constexpr int kBN = BN;
    static constexpr int kBRows = BN / 2;                 // B rows per CTA
    static constexpr int kUnits = 2;                      // scale units per row group per chunk
    static constexpr int kMmas = 4;                       // K=64 MMAs per chunk
    static constexpr int kABytes = kBM * kCB;
    static constexpr int kBBytes = kBRows * kCB;
    static constexpr int kSfaBytes = kUnits * kSfUnit;
    static constexpr int kSfbBytes = 2 * kUnits * kSfUnit;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr uint32_t kPairTx = 2u * uint32_t(kStageBytes);   // both CTAs' bytes of a stage
    // scale columns of a k-unit: A's unit at +0, B's two units at +4 and +8
    static constexpr uint32_t kSfUnitCols = 12;
    static constexpr uint32_t kSfStageCols = kSfUnitCols * kUnits;
    static constexpr int kOutBytes = 2 * 2048;            // a warp's two 2 KB output boxes
    static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (1u << 23) |
                                       (uint32_t(256 >> 4) << 24);
    static constexpr int kEpiCols = BN / 2;
    static constexpr size_t kRing = size_t(ST) * kStageBytes;
    static constexpr int kAccBufs = (2 * BN + ST * int(kSfStageCols) <= kTmemCols) ? 2 : 1;
    static constexpr uint32_t kSfCol = uint32_t(kAccBufs * BN);
    static constexpr size_t kSmem = kRing + size_t(kEpiWarps) * kOutBytes + 1024 + (3 * ST + 6) * sizeof(uint64_t) + 16;
    static_assert(BN == 256 || BN == 192, "tile columns");
    static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0 && kStageBytes % 1024 == 0,
                  "operands and stages keep the 1 KB alignment of the 128-byte swizzle");
    static_assert(kSfCol + ST * kSfStageCols <= kTmemCols, "tensor memory columns");
    static_assert(kSmem <= kSmemMax, "shared memory");
};

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_count_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// The shared::cluster address of the variable at shared::cta address `addr`
// in the cluster's CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Every thread of both CTAs (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Arrive on an mbarrier of either CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// TMA loads into this CTA's shared memory whose bytes complete on `bar`, an
// mbarrier of either CTA of the pair (here the leader's).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, int32_t x, int32_t y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, int32_t x, int32_t y, int32_t z,
                                                 uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void umma_mxf4_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t id,
                                               uint32_t tmem_sfa, uint32_t tmem_sfb, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                     tmem_d),
                 "l"(adesc), "l"(bdesc), "r"(id), "r"(accumulate), "r"(tmem_sfa), "r"(tmem_sfb)
                 : "memory");
}

// One 512-byte scale unit of each CTA's shared memory (same address in both)
// to the same 4 columns of its own tensor memory, replicated to the four
// 32-lane quarters.
__device__ __forceinline__ void tmem_copy_unit_pair(uint32_t taddr, uint32_t saddr)
{
    const uint64_t desc = mma::smem_desc(saddr, 128, 0);
    asm volatile("{\n\t.reg .pred e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr), "l"(desc) : "memory");
}

// Arrive on `bar` (shared::cluster, either CTA) when every tcgen05 operation
// this thread issued so far has completed on both SMs.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar)
{
    asm volatile("{\n\t.reg .pred e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
                 : "memory");
}

template <class C, bool F32OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mxf4_gemm_pair_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap b_map,
                      const __grid_constant__ CUtensorMap asf_map, const __grid_constant__ CUtensorMap bsf_map,
                      const __grid_constant__ CUtensorMap out_map, void *__restrict__ out, int M, int N, int K,
                      long long budget)
{
    pdl_wait();
    constexpr int ST = C::kST;
    constexpr int kBN = C::kBN;
    constexpr int NA = C::kAccBufs;
    constexpr bool kStaged = !F32OUT;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t *stage_out = base + C::kRing;                // [kEpiWarps] x 4 KB output staging
    uint64_t *bars = reinterpret_cast<uint64_t *>(stage_out + size_t(kEpiWarps) * C::kOutBytes);
    uint64_t *full = bars;                    // [ST] (leader) both CTAs' copies of the stage landed
    uint64_t *empty = bars + ST;              // [ST] MMAs reading the stage done (leader's commit)
    uint64_t *sf_ready = bars + 2 * ST;       // [ST] (leader) the stage's scale units are in both tensor memories
    uint64_t *acc_full = bars + 3 * ST;       // [2] accumulator b holds a finished tile (leader's commit)
    uint64_t *acc_empty = acc_full + 2;       // [2] (leader) accumulator b read by both CTAs' 16 epilogue warps
    uint64_t *done = acc_full + 4;            // every MMA of the pair completed (leader's final commit)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 6);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();   // 0: the leader
    const int cid = int(cluster_id_x()), ncl = int(cluster_count_x());

    const int MT = (M + 2 * kBM - 1) / (2 * kBM);
    const int NT = (N + kBN - 1) / kBN;
    const int tiles = MT * NT;
    const int KC = (K + 2 * C::kCB - 1) / (2 * C::kCB);   // k-chunks
    const int KS = (K + 63) / 64;                         // MMA K steps

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_ready[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * kEpiWarps);
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    mma::tc_fence_before();
    cluster_sync();                           // both CTAs' barriers initialised, tensor memory allocated
    mma::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        {
            // ---------------- producer (both CTAs; the whole warp, one elected lane issues)
            const uint32_t lead_full = cluster_addr(smem_addr(full), 0);
            int k = 0, filled = 0;
            bool ok = true;
            for (int t = cid; t < tiles && ok; t += ncl) {
                const int mt = t / NT, nt = t % NT;
                const int row_a = mt * 2 * kBM + int(rank) * kBM;
                const int row_b = nt * kBN + int(rank) * C::kBRows;
                const int ga = 2 * mt + int(rank);           // this CTA's A row group
                const int gb = nt * kBN / 128;               // the tile's first B row group
                for (int c = 0; c < KC; ++c, ++k) {
                    const int s = k % ST;
                    if (k >= ST && !warp_wait(&empty[s], ((k / ST) - 1) & 1, budget)) {
                        if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                        ok = false;
                        break;
                    }
                    uint8_t *st = base + size_t(s) * C::kStageBytes;
                    uint8_t *sfa = st + C::kABytes + C::kBBytes;
                    uint8_t *sfb = sfa + C::kSfaBytes;
                    const uint32_t bar = lead_full + uint32_t(s) * 8;
                    if (elect_one()) {
                        if (rank == 0) mbar_expect_tx(&full[s], C::kPairTx);
                        tma_load_2d_pair(st, &a_map, c * C::kCB, row_a, bar);
                        tma_load_2d_pair(st + C::kABytes, &b_map, c * C::kCB, row_b, bar);
                        // scale units 2c, 2c + 1 = 256-byte rows 4c .. 4c + 3 of the row group
                        tma_load_3d_pair(sfa, &asf_map, 0, 4 * c, ga, bar);
                        tma_load_3d_pair(sfb, &bsf_map, 0, 4 * c, gb, bar);
                    }
                    __syncwarp();
                    filled = k + 1;
                }
            }
            // drain: every copy issued has landed (the leader's barriers count
            // both CTAs' bytes) and the MMAs reading this CTA's stages have
            // completed (their commits have arrived) before the CTA may exit
            const int k0 = filled > ST ? filled - ST : 0;
            if (rank == 0)
                for (int kk = k0; kk < filled; ++kk)
                    if (!warp_wait(&full[kk % ST], (kk / ST) & 1, budget)) {
                        if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                        break;
                    }
            for (int kk = k0; kk < filled; ++kk)
                if (!warp_wait(&empty[kk % ST], (kk / ST) & 1, budget)) {
                    if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
        }
    } else if (warp == 1) {
        if (rank == 0) {
            // ---------------- MMAs (the leader's warp; one elected lane issues)
            const uint32_t empty0 = cluster_addr(smem_addr(empty), 0), empty1 = cluster_addr(smem_addr(empty), 1);
            const uint32_t accf0 = cluster_addr(smem_addr(acc_full), 0), accf1 = cluster_addr(smem_addr(acc_full), 1);
            int k = 0, it = 0;
            bool ok = true;
            for (int t = cid; t < tiles && ok; t += ncl, ++it) {
                // a 192-column tile starting mid-unit: the MMA reads B's scales
                // off = 0 or 2 columns (32-row groups) into the first unit
                const uint32_t off = uint32_t(((t % NT) * kBN % 128) / 32);
                const int ab = it % NA;
                if (it >= NA && !warp_wait(&acc_empty[ab], ((it / NA) - 1) & 1, budget)) {
                    if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                    break;
                }
                mma::tc_fence_after();
                for (int c = 0; c < KC; ++c, ++k) {
                    const int s = k % ST;
                    if (!warp_wait(&full[s], (k / ST) & 1, budget) || !warp_wait(&sf_ready[s], (k / ST) & 1, budget)) {
                        if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                        ok = false;
                        break;
                    }
                    mma::tc_fence_after();
                    const uint32_t a0 = smem_addr(base + size_t(s) * C::kStageBytes);
                    const uint32_t b0 = a0 + C::kABytes;
                    const uint32_t tsf = tmem_base + C::kSfCol + uint32_t(s) * C::kSfStageCols;
#pragma unroll
                    for (int j = 0; j < C::kMmas; ++j) {
                        if (c * C::kMmas + j >= KS) break;
                        const uint32_t sf_id = 2 * (j & 1);
                        const uint32_t u = j >> 1;
                        const uint64_t ad = mma::smem_desc(a0 + j * 32, 8 * C::kCB, mma::kLayoutSw128);
                        const uint64_t bd = mma::smem_desc(b0 + j * 32, 8 * C::kCB, mma::kLayoutSw128);
                        const uint32_t tu = tsf + C::kSfUnitCols * u;
                        umma_mxf4_pair(tmem_base + kAccCol + uint32_t(ab * kBN), ad, bd, idesc(C::kIdesc, sf_id),
                                       tu | (sf_id << 30), (tu + 4 + off) | (sf_id << 30), (c | j) != 0);
                    }
                    umma_commit_pair(empty0 + uint32_t(s) * 8);
                    umma_commit_pair(empty1 + uint32_t(s) * 8);
                }
                if (!ok) break;
                umma_commit_pair(accf0 + uint32_t(ab) * 8);
                umma_commit_pair(accf1 + uint32_t(ab) * 8);
            }
            // every MMA issued has completed before the tensor memory is freed
            umma_commit_pair(cluster_addr(smem_addr(done), 1));
            umma_commit_pair(cluster_addr(smem_addr(done), 0));
            if (!warp_wait(done, 0, budget) && lane == 0) atomicAdd(&g_wait_timeouts, 1);
        } else {
            // the peer: the leader's final commit has arrived here too
            if (!warp_wait(done, 0, budget) && lane == 0) atomicAdd(&g_wait_timeouts, 1);
        }
    } else if (warp == kCopyWarp) {
        if (rank == 0) {
            // ---------------- scale copies (the leader's warp): each
            // CTA's units of the stage to its own tensor memory
            int k = 0, issued = 0;
            bool ok = true;
            for (int t = cid; t < tiles && ok; t += ncl) {
                for (int c = 0; c < KC; ++c, ++k) {
                    const int s = k % ST;
                    if (!warp_wait(&full[s], (k / ST) & 1, budget)) {
                        if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                        ok = false;
                        break;
                    }
                    mma::tc_fence_after();
                    const uint32_t sfa = smem_addr(base + size_t(s) * C::kStageBytes) + C::kABytes + C::kBBytes;
                    const uint32_t sfb = sfa + C::kSfaBytes;
                    const uint32_t tsf = tmem_base + C::kSfCol + uint32_t(s) * C::kSfStageCols;
#pragma unroll
                    for (int u = 0; u < C::kUnits; ++u) {
                        const uint32_t tu = tsf + C::kSfUnitCols * u;
                        tmem_copy_unit_pair(tu, sfa + u * kSfUnit);
                        tmem_copy_unit_pair(tu + 4, sfb + u * kSfUnit);
                        tmem_copy_unit_pair(tu + 8, sfb + (C::kUnits + u) * kSfUnit);
                    }
                    umma_commit_pair(smem_addr(&sf_ready[s]));
                    issued = k + 1;
                }
            }
            if (issued > 0 && !warp_wait(&sf_ready[(issued - 1) % ST], ((issued - 1) / ST) & 1, budget) && lane == 0)
                atomicAdd(&g_wait_timeouts, 1);
        }
    } else {
        // ---------------- epilogue (both CTAs, own accumulator lanes)
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const uint32_t lead_acc_empty = cluster_addr(smem_addr(acc_empty), 0);
        int it = 0, nbox = 0;
        for (int t = cid; t < tiles; t += ncl, ++it) {
            const int mt = t / NT, nt = t % NT;
            const int ab = it % NA;
            const bool ready = mbar_wait(&acc_full[ab], (it / NA) & 1, budget);
            if (!__all_sync(0xffffffffu, ready)) {
                if (lane == 0) atomicAdd(&g_wait_timeouts, 1);
                break;
            }
            mma::tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + kAccCol + uint32_t(ab * kBN + h * C::kEpiCols);
            epilogue_tile<C::kEpiCols, F32OUT, kStaged, true>(
                taddr, mt * 2 * kBM + int(rank) * kBM + q * 32, nt * kBN + h * C::kEpiCols, M, N, out, &out_map,
                stage_out + size_t(warp - 2) * C::kOutBytes,
                [&] { mbar_arrive_cluster(lead_acc_empty + uint32_t(ab) * 8); }, &nbox);
        }
        if constexpr (kStaged) {
            if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        }
    }

    mma::tc_fence_before();
    __syncwarp();
    cluster_sync();
    if (warp == 1) {
        mma::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// Configurations (mxf4_gemm_variant): 1 = 128-byte chunks, 4 stages, stores
// from registers; 2 = 64-byte chunks, 6 stages, TMA-store epilogue; 3 = 64, 4,
// TMA stores; 4 = 128, 3, TMA stores; 5 = 64, 8, stores from registers;
// 6 = as 4 with 192-column tiles.
using Cfg1 = Cfg<128, 4, false>;
using Cfg2 = Cfg<64, 6, true>;
using Cfg3 = Cfg<64, 4, true>;
using Cfg4 = Cfg<128, 3, true>;
using Cfg5 = Cfg<64, 8, false>;
using Cfg6 = Cfg<128, 3, true, 192>;
// The SM-pair form: 7 = 256 x 256 tiles, 5 stages, one accumulator;
// 8 = 256 x 192 tiles, 5 stages, two accumulators.
using Pair7 = PairCfg<256, 5>;
using Pair8 = PairCfg<192, 5>;

}  // namespace gemm
