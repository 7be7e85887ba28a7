// gemm_sm100.cu -- block-scaled NVFP4 GEMM on the 5th-generation tensor cores (sm_100a).
//
// D[M][N] = s_tA * s_tB * sum_k (qA[m][k] * sA[m][k/16]) * (qB[n][k] * sB[n][k/16])
// with E2M1 codes q, E4M3 block scales s and fp32 tensor scales s_t (gist.science "Pretraining
// Large Language Models with NVFP4", 2.A; the FP4 GEMMs of the linear layers are the hot
// spot, brainai.pro "Details techniques").
//
// Two kernels.  For M >= 256 the launcher runs the SM-pair kernel further below (256 x 256 tiles
// on two SMs: fewer operand bytes per SM per K block, a five-stage ring); the 1-SM kernel here
// serves smaller M (and every shape under NVFP4_GEMM_VARIANT=1sm).
//
// 1-SM kernel.  Persistent: one CTA per SM walks 128 x 256 output tiles (bands of 8 tile rows or columns that
// sweep the smaller operand, for L2 reuse: tile_coords); the shared-memory ring runs on across
// tiles:
//   warp 0      TMA producer: per 256-wide K block, the A tile (128 rows x 128 bytes) and the
//               B tile (256 x 128 bytes) by cp.async.bulk.tensor with 128-byte swizzle, and the
//               matching 512-byte scale tiles by cp.async.bulk, into a 4-stage ring;
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma kind::mxf4nvf4
//               block_scale scale_vec::4X (M=128, N=256, K=64), accumulating in fp32 in TMEM;
//               tcgen05.commit frees the stage;
//   last 4 warps write each stage's scale tiles from shared memory into TMEM with tcgen05.st
//               (one warp per TMEM lane quadrant).  Moving the scales with tcgen05.cp instead
//               costs more tensor-pipe time than the MMAs themselves (measured: 12 copies per
//               256-wide K block take ~790 cycles and serialise with the 512 cycles of MMAs;
//               the tcgen05.st path takes ~60 cycles and overlaps them);
//   warps 2-17  epilogue: four warps per TMEM lane quadrant, 64 columns each, read the
//               accumulator into registers (tcgen05.ld 32x32b), release it to the MMA warp, then
//               scale by s_tA*s_tB and store bf16 or fp32 -- overlapping the next tile's MMAs
//               (measured: storing before the release stalled the MMAs ~5000 cycles per tile);
// TMEM columns: [0, 256) accumulator; per stage s, [256 + 48 s, +16) scales of A (4 columns per
// 64-wide K step), [+16, +48) scales of B (8 columns per K step: two 128-row tiles).  A stage's
// scale columns are rewritten only after its smem slot was refilled, i.e. after the MMAs that
// read them completed (tcgen05.commit -> empty -> producer -> full).
// Every mbarrier wait is bounded by a cycle budget; on expiry the CTA raises the timeout
// flag, drains its copies and MMAs (again bounded) and frees its TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "nvfp4_device.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {

constexpr int kBM = 128, kBN = 256, kBK = 256;  // K in elements (128 bytes of codes)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK / 2;                 // 16384
constexpr int kBBytes = kBN * kBK / 2;                 // 32768
constexpr int kSFABytes = (kBM / 128) * (kBK / 64) * 512;  // 2048
constexpr int kSFBBytes = (kBN / 128) * (kBK / 64) * 512;  // 4096
constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;  // 55296 (54 KiB)
constexpr int kBarrierBytes = 512;
constexpr int kStoreSlots = 2;                         // output staging for the TMA stores
constexpr int kStoreSlotBytes = 32 * 128;              // 32 rows x 128 bytes, 128-byte swizzle
constexpr int kGemmSmem = kStages * kStageBytes + kStoreSlots * kStoreSlotBytes + kBarrierBytes + 1024;  // + alignment slack
static_assert(kGemmSmem <= 232448, "1-SM kernel shared memory");
constexpr int kGemm1Threads = 704;  // producer, MMA, 16 epilogue warps, 4 scale warps (both kernels)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 256, kSfColsPerStage = 48;

static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment for the 128B swizzle");
static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");

// instruction descriptor: dense, A/B = E2M1 (format 1 of the mxf4 kinds), both K-major,
// N >> 3 at bit 17, scale type UE4M3 (bit 23 = 0), M >> 4 at bit 24, scale ids 0
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

// Budget of the teardown waits (copies and MMAs still in flight after an abort).  Fixed, not the
// caller's budget: however small that is, no CTA exits (or frees TMEM) before its own copies have
// landed and its MMAs have completed.
constexpr uint64_t kDrainBudgetNs = 2000000000ull;

// ---------------------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t cycles() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
    return t;
}

// Bounded wait.  Returns false if the CTA aborted (another role timed out) or this wait ran out
// of its budget (then it raises the abort and the timeout flag).  `honor_abort` = false is used
// by the drain after an abort, which must still see copies land.  The budget is counted in SM
// cycles (2 per nanosecond, i.e. an upper bound for clocks <= 2 GHz); the cycle counter is read
// only after a burst of polls, so a wait that succeeds quickly costs no timer read.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                          uint32_t* flags, uint64_t budget_ns, bool honor_abort = true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = cycles(), limit = 2 * budget_ns;
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (honor_abort && *abort) return false;
        if (cycles() - t0 > limit) {
            *abort = 1u;
            atomicOr(flags, kFlagTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.b32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups 1024 bytes apart
// (stride byte offset), leading byte offset unused (1), descriptor version 1 (bit 46),
// layout type 2 = SWIZZLE_128B (bits 61-63)
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}
// tcgen05.st of 16 / 32 consecutive 32-bit columns of this warp's 32 TMEM lanes
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// MXFP4 operands (blocks of 32, UE8M0 scales): two scales per row per K=64 step
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Operand format of a GEMM instantiation.  Every format stages 128-byte rows of A and B per
// pipeline stage and consumes 32 bytes of each row per MMA (four MMAs per stage):
//   NVFP4: E2M1 with E4M3 scales per 16 elements, a 512-byte scale tile (128 rows x 4 scales) per
//          64-wide K step (K = 64 per MMA);
//   MXFP4: E2M1 with UE8M0 scales per 32 elements, a tile per 128-wide K step, read by two K=64
//          MMAs: the instruction descriptor's scale-factor IDs (bits 29-30 for A, 4-5 for B) pick
//          bytes 0-1 or 2-3 of each 32-bit TMEM scale word;
//   BF16:  no scales, kind::f16 with K = 16 per MMA (the high-precision layers' path).
enum : int { kNVF4 = 0, kMXF4 = 1, kBF16 = 2 };
template <int F>
struct OpFmt {
    static constexpr int kTilesPerBlock = F == kNVF4 ? 4 : F == kMXF4 ? 2 : 0;   // scale tiles per stage
    __device__ static __forceinline__ int tile_of_step(int j) { return F == kMXF4 ? (j >> 1) : j; }
    __device__ static __forceinline__ uint32_t idesc(uint32_t base, int j) {
        if (F != kMXF4) return base;
        const uint32_t id = 2u * (uint32_t)(j & 1);
        return base | (1u << 23) | (id << 29) | (id << 4);
    }
};

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// shared -> global tile store by the TMA (clipped at the tensor bounds), in this thread's bulk group
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
// shared -> global tile reduce-add by the TMA (fp32 add into the destination), in this thread's
// bulk group
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------------------------------
// the kernel: persistent, one CTA per SM, static tile schedule
// ---------------------------------------------------------------------------------------
struct GemmParams {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* sta;
    const float* stb;
    void* d;
    int64_t ldd;
    int32_t out_fp32;
    int32_t M, N, K;
    int32_t nkt;            // scale tiles per 128-row tile along K: ceil(K / 64) (NVFP4), ceil(K / 128) (MXFP4)
    int32_t kst;            // ceil(K / 64): 64-wide K steps (MMAs per row of tiles)
    int32_t num_kb;         // ceil(K / 256): pipeline stages' worth of K per tile
    int32_t sfb_row_tiles;  // ceil(N / 128)
    int32_t sfa_row_tiles;  // ceil(M / 128)
    int32_t tiles_m, tiles_n;
    int32_t group_n;        // raster: 1 = groups of kGroup N tiles sweep all M tiles, 0 = the transpose
    uint32_t* flags;
    uint64_t budget_ns;
    // reduce-scatter epilogue (0 owners: plain stores to D): output rows [o * owner_rows,
    // (o + 1) * owner_rows) are added into owner o's shard through its own tensor map
    int32_t n_owners;
    int32_t owner_rows;
    // amax epilogue (null: off; bf16 output): the plain amax of the stored output and the amax of
    // its 16-point RHT along the rows go to amax_out[0] and amax_out[1] (fp32 bits, atomic max)
    uint32_t* amax_out;
    uint32_t rht_mask[16];   // row i of a 16-row group: 0x80008000 where the RHT sign is -1
};

// The shards of a reduce-scatter epilogue: one fp32 output map per owner (a local buffer or
// another GPU's, through its peer address)
constexpr int kMaxOwners = 8;
struct OwnerMaps {
    CUtensorMap m[kMaxOwners];
};

constexpr int kEpi1Warps = 16;                     // four warps per TMEM lane quadrant, 64 columns each
constexpr int kSfWarps = 4;                        // one warp per TMEM lane quadrant
constexpr int kGroup = 8;                          // L2 raster: tiles of 8 rows (or columns) of tiles swept together

// tile index -> (m tile, n tile).  The output is cut into bands of kGroup tile rows (group_n = 0)
// or tile columns (group_n = 1); the CTAs walk a band across, column by column (row by row), so
// the band's tiles of one operand stay in L2 while the other operand is swept.  The host picks the
// orientation that sweeps the smaller operand; alternate bands sweep in opposite directions so the
// first tiles of a sweep are the last ones of the previous sweep, still in L2.
__device__ __forceinline__ void tile_coords(int t, const GemmParams& p, int& tm, int& tn) {
    const int band_len = p.group_n ? p.tiles_m : p.tiles_n;     // tiles along the sweep
    const int nbands_dim = p.group_n ? p.tiles_n : p.tiles_m;   // tiles across the bands
    const int per_band = kGroup * band_len;
    const int g = t / per_band, r = t - g * per_band;
    const int w = min(kGroup, nbands_dim - g * kGroup);         // width of this band (last may be narrow)
    int along = r / w;
    const int across = g * kGroup + (r - along * w);
    if (g & 1) along = band_len - 1 - along;
    if (p.group_n) {
        tm = along;
        tn = across;
    } else {
        tm = across;
        tn = along;
    }
}

// Writes one epilogue warp's 32 rows x 64 accumulator columns (r: two 32-column chunks of fp32
// bits) to D through the TMA, scaled by alpha: 128-byte-wide boxes (64 bf16 or 32 fp32 columns x
// 32 rows) staged in kSlots swizzled 4 KiB shared-memory slots, taken in a fixed order.  Box b of
// a tile (b = warp for bf16, 2 x warp + half for fp32) uses slot b % kSlots once box b - kSlots
// has been read by its store; the last boxes of a tile hand over to the first ones of the next.
// One mbarrier per box position keeps every waiting warp at most one phase ahead of it.  Returns
// false on abort.
// With owner maps (the reduce-scatter epilogue) each box is added into the shard of the owner of
// its rows instead of stored.
// With p.amax_out (bf16 output) the warp also reads its staged box back, each lane one column pair
// of both 16-row groups (box_read: 32 shared loads, after which the slot can be released), and
// then takes the plain and RHT amax of those words (words_amax), excluding rows >= M and columns
// >= N, which hold padding: the same sign flips, butterfly and maxima as the amax pass of a
// quantize call over the stored tensor.
__device__ __forceinline__ void box_read(uint32_t sbase, uint32_t (&w)[2][16]) {
    const uint32_t lane = threadIdx.x & 31;
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t rr = (uint32_t)(16 * g + i);
            asm volatile("ld.shared.u32 %0, [%1];"
                         : "=r"(w[g][i])
                         : "r"(sbase + rr * 128u + (((lane >> 2) ^ (rr & 7u)) << 4) + ((lane & 3u) << 2)));
        }
}
__device__ __forceinline__ void words_amax(const uint32_t (&w)[2][16], int x, int y, const GemmParams& p,
                                           uint32_t& am_plain, float& am_rht) {
    const int col = x + 2 * (threadIdx.x & 31);
    if (col >= p.N) return;
    const uint32_t keep = col + 1 < p.N ? 0xFFFFFFFFu : 0x0000FFFFu;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        if (y + 16 * g >= p.M) break;
        uint64_t f[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t v = w[g][i] & keep;
            am_plain = __vmaxu2(am_plain, v & 0x7FFF7FFFu);
            f[i] = bf16x2_to_f2(v ^ p.rht_mask[i]);
        }
        rht16_pairs(f);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            float a0, a1, b0, b1;
            f2_split(f[i], a0, a1);
            f2_split(f[i + 1], b0, b1);
            am_rht = max3_abs(max3_abs(am_rht, a0, a1), b0, b1);
        }
    }
}

// The amax epilogue's per-warp maxima into the output words (and the non-finite flag)
__device__ __forceinline__ void amax_flush(const GemmParams& p, uint32_t am_plain, float am_rht) {
    uint32_t m = max(am_plain & 0xFFFFu, am_plain >> 16) << 16;
    uint32_t mr = __float_as_uint(am_rht);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        mr = max(mr, __shfl_xor_sync(0xFFFFFFFFu, mr, o));   // non-negative floats order as integers
    }
    if ((threadIdx.x & 31) == 0) {
        if (m) atomicMax(p.amax_out, m);
        if (mr) atomicMax(p.amax_out + 1, mr);
        if (m >= 0x7F800000u || mr >= 0x7F800000u) atomicOr(p.flags, kFlagNonFinite);
    }
}

template <int kSlots, bool AMAX>
__device__ __forceinline__ bool store_boxes(const CUtensorMap* tmD, const CUtensorMap* owner_maps, uint8_t* store_area,
                                            uint64_t* boxgo_bar, const uint32_t (&r)[2][32], int ew, int local, int x0,
                                            int y, const GemmParams& p, float alpha, volatile uint32_t* abort_flag,
                                            uint32_t& am_plain, float& am_rht) {
    const int lane = threadIdx.x & 31;
    const int nbox = (!AMAX && p.out_fp32) ? 2 : 1;   // the amax epilogue serves bf16 outputs only
    const int nb = kEpi1Warps * nbox;   // boxes per tile, a multiple of kSlots
    const uint32_t swz = (uint32_t)(lane & 7);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (h >= nbox) break;
        const int b = ew * nbox + h;
        const uint32_t slot = (uint32_t)(b % kSlots);
        bool free_ok = true;
        if (b >= kSlots || local > 0)   // the n-th completion of a barrier is waited with parity n & 1
            free_ok = mbar_wait(smem_u32(&boxgo_bar[b]), (uint32_t)(b >= kSlots ? local : local - 1) & 1u, abort_flag,
                                p.flags, p.budget_ns);
        if (!__all_sync(0xFFFFFFFFu, free_ok)) return false;
        const uint32_t sbase = smem_u32(store_area + slot * kStoreSlotBytes);
        const uint32_t srow = sbase + (uint32_t)lane * 128u;
        int x;
        if (p.out_fp32) {
            x = x0 + h * 32;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_shared_v4(srow + (((uint32_t)c ^ swz) << 4), __float_as_uint(__fmul_rn(__uint_as_float(r[h][4 * c]), alpha)),
                             __float_as_uint(__fmul_rn(__uint_as_float(r[h][4 * c + 1]), alpha)),
                             __float_as_uint(__fmul_rn(__uint_as_float(r[h][4 * c + 2]), alpha)),
                             __float_as_uint(__fmul_rn(__uint_as_float(r[h][4 * c + 3]), alpha)));
        } else {
            x = x0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = 8 * c + 2 * e;   // 0..62 within the warp's 64 columns
                    const float lo = __fmul_rn(__uint_as_float(r[col >> 5][col & 31]), alpha);
                    const float hi = __fmul_rn(__uint_as_float(r[col >> 5][(col & 31) + 1]), alpha);
                    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[e]) : "f"(hi), "f"(lo));
                }
                st_shared_v4(srow + (((uint32_t)c ^ swz) << 4), w[0], w[1], w[2], w[3]);
            }
        }
        fence_async_smem();
        __syncwarp();
        if (AMAX) {
            // the store first, then the read-back of the box and its release, then the maxima
            if (lane == 0 && x < p.N && y < p.M) tma_store_2d(tmD, sbase, x, y);
            if (lane == 0) bulk_commit();
            uint32_t wv[2][16];
            box_read(sbase, wv);
            __syncwarp();
            if (lane == 0) {
                bulk_wait_read_all();
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&boxgo_bar[(b + kSlots) % nb]))
                             : "memory");
            }
            __syncwarp();
            words_amax(wv, x, y, p, am_plain, am_rht);
            continue;
        }
        if (lane == 0) {
            if (x < p.N && y < p.M) {
                if (owner_maps) {
                    const int o = y / p.owner_rows;
                    tma_reduce_add_2d(&owner_maps[o], sbase, x, y - o * p.owner_rows);
                } else {
                    tma_store_2d(tmD, sbase, x, y);
                }
            }
            bulk_commit();
            bulk_wait_read_all();
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&boxgo_bar[(b + kSlots) % nb])) : "memory");
        }
        __syncwarp();
    }
    return true;
}

template <bool MX, bool AMAX>
__global__ void __launch_bounds__(kGemm1Threads, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmD, const __grid_constant__ OwnerMaps om, GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* store_area = smem + kStages * kStageBytes;
    uint8_t* bar_area = store_area + kStoreSlots * kStoreSlotBytes;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(bar_area);
    uint64_t* empty_bar = full_bar + kStages;
    uint64_t* sfready_bar = empty_bar + kStages;   // stage's scales written into TMEM (scale warps -> MMA)
    uint64_t* tfull_bar = sfready_bar + kStages;   // accumulator ready (MMA -> epilogue)
    uint64_t* tempty_bar = tfull_bar + 1;          // accumulator drained (epilogue -> MMA)
    uint64_t* done_bar = tempty_bar + 1;
    uint64_t* boxgo_bar = done_bar + 1;            // store slot hand-over, one per box position (store_boxes)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(boxgo_bar + 2 * kEpi1Warps);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = p.tiles_m * p.tiles_n;

    for (int i = threadIdx.x; i < kStages * (kSFABytes + kSFBBytes) / 16; i += kGemm1Threads) {
        const int s = i / ((kSFABytes + kSFBBytes) / 16), o = i % ((kSFABytes + kSFBBytes) / 16);
        reinterpret_cast<uint4*>(smem + s * kStageBytes + kABytes + kBBytes)[o] = make_uint4(0, 0, 0, 0);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
            mbar_init(smem_u32(&sfready_bar[s]), kSfWarps);
        }
        mbar_init(smem_u32(tfull_bar), 1);
        mbar_init(smem_u32(tempty_bar), kEpi1Warps);
        mbar_init(smem_u32(done_bar), 1);
        for (int k = 0; k < 2 * kEpi1Warps; ++k) mbar_init(smem_u32(&boxgo_bar[k]), 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------- producer -------------------------------------------
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
            int g = 0;   // stages issued, across tiles
            bool ok = true;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, p, tm, tn);
                const int m0 = tm * kBM, n0 = tn * kBN;
                for (int kb = 0; kb < p.num_kb; ++kb, ++g) {
                    const int s = g % kStages;
                    const uint32_t ph = (uint32_t)(g / kStages) & 1u;
                    if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag, p.flags, p.budget_ns)) {
                        ok = false;
                        break;
                    }
                    constexpr int tpb = OpFmt<MX ? kMXF4 : kNVF4>::kTilesPerBlock;
                    const int tiles = min(tpb, p.nkt - tpb * kb);
                    const uint32_t sf_bytes = (uint32_t)tiles * 512u;
                    int btiles = 0;
                    for (int u = 0; u < 2; ++u) btiles += ((n0 >> 7) + u < p.sfb_row_tiles) ? 1 : 0;
                    const uint32_t full = smem_u32(&full_bar[s]);
                    mbar_expect_tx(full, (uint32_t)(kABytes + kBBytes) + sf_bytes * (uint32_t)(1 + btiles));
                    uint8_t* st = smem + s * kStageBytes;
                    tma_load_2d(smem_u32(st), &tmA, kb * 128, m0, full);
                    tma_load_2d(smem_u32(st + kABytes), &tmB, kb * 128, n0, full);
                    bulk_load(smem_u32(st + kABytes + kBBytes), p.sfa + ((int64_t)(m0 >> 7) * p.nkt + tpb * kb) * 512,
                              sf_bytes, full);
                    for (int u = 0; u < 2; ++u) {
                        const int rt = (n0 >> 7) + u;
                        if (rt < p.sfb_row_tiles)
                            bulk_load(smem_u32(st + kABytes + kBBytes + kSFABytes + u * 2048),
                                      p.sfb + ((int64_t)rt * p.nkt + tpb * kb) * 512, sf_bytes, full);
                    }
                }
            }
            // drain: every copy this thread issued lands before the CTA exits.  Stages before
            // g - kStages were consumed (their slots were refilled); after a normal run the last
            // kStages were consumed too and these waits return at once.
            for (int k = max(0, g - kStages); k < g; ++k)
                mbar_wait(smem_u32(&full_bar[k % kStages]), (uint32_t)(k / kStages) & 1u, abort_flag, p.flags,
                          kDrainBudgetNs, false);
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -----------------------------------------
        // The whole warp runs the loop and waits (warp-uniform control flow keeps the MMA
        // operands uniform); one elected lane issues the MMAs and commits.
        const uint32_t sbase = smem_u32(smem);
        const uint64_t adesc0 = desc_k_sw128(sbase), bdesc0 = desc_k_sw128(sbase + kABytes);
        int g = 0, local = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
            // the epilogue must have drained the previous tile's accumulator
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(tempty_bar), ((uint32_t)local & 1u) ^ 1u, abort_flag, p.flags,
                                                   p.budget_ns)))
                break;
            tc_fence_after();
            for (int kb = 0; kb < p.num_kb; ++kb, ++g) {
                const int s = g % kStages;
                const uint32_t ph = (uint32_t)(g / kStages) & 1u;
                const bool landed = mbar_wait(smem_u32(&full_bar[s]), ph, abort_flag, p.flags, p.budget_ns) &&
                                    mbar_wait(smem_u32(&sfready_bar[s]), ph, abort_flag, p.flags, p.budget_ns);
                if (!__all_sync(0xFFFFFFFFu, landed)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int steps = min(4, p.kst - 4 * kb);
                // descriptors advance by the stage offset and 32 bytes per K step (address field >> 4)
                const uint64_t aoff = (uint64_t)((s * kStageBytes) >> 4);
                const uint32_t t_sfa = tmem + kSfCol0 + s * kSfColsPerStage;
                if (elect_one()) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (j < steps) {
                            const int tj = OpFmt<MX ? kMXF4 : kNVF4>::tile_of_step(j);
                            if (MX)
                                mma_mxf4(tmem, adesc0 + aoff + 2 * j, bdesc0 + aoff + 2 * j, OpFmt<MX ? kMXF4 : kNVF4>::idesc(kIdesc, j),
                                         t_sfa + 4 * tj, t_sfa + 16 + 8 * tj, (kb | j) != 0 ? 1u : 0u);
                            else
                                mma_nvf4(tmem, adesc0 + aoff + 2 * j, bdesc0 + aoff + 2 * j, kIdesc, t_sfa + 4 * tj,
                                         t_sfa + 16 + 8 * tj, (kb | j) != 0 ? 1u : 0u);
                        }
                    mma_commit(smem_u32(&empty_bar[s]));
                }
                __syncwarp();
            }
            if (ok && elect_one()) mma_commit(smem_u32(tfull_bar));
            __syncwarp();
        }
        // all MMAs of this warp complete before TMEM may be freed
        if (elect_one()) mma_commit(smem_u32(done_bar));
        __syncwarp();
        mbar_wait(smem_u32(done_bar), 0u, abort_flag, p.flags, kDrainBudgetNs, false);
    } else if (warp < 2 + kEpi1Warps) {
        // ------------------------------- epilogue (warps 2..17) -----------------------------
        // Each warp owns 32 accumulator rows (its TMEM lane quadrant) x 64 columns.  It reads
        // both 32-column chunks, releases the accumulator to the MMA warp, then scales and
        // converts in registers and hands its boxes to the TMA (store_boxes).  Plain st.global of the rows
        // (32 lines per instruction) held up the MMA and scale warps' shared-memory traffic for
        // thousands of cycles per tile; the TMA store leaves that path nearly idle.
        const int ew = warp - 2;
        const int q = warp & 3;
        const int cq = ew >> 2;                 // which 64 of the 256 accumulator columns
        const float alpha = p.sta ? __fmul_rn(*p.sta, *p.stb) : 1.0f;   // MXFP4: no tensor scales
        int local = 0;
        bool ok = true;
        uint32_t am_plain = 0;
        float am_rht = 0.0f;
        for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
            int tm, tn;
            tile_coords(t, p, tm, tn);
            const bool full = mbar_wait(smem_u32(tfull_bar), (uint32_t)local & 1u, abort_flag, p.flags, p.budget_ns);
            if (!__all_sync(0xFFFFFFFFu, full)) break;
            tc_fence_after();
            uint32_t r[2][32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cq * 64), r[0]);
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cq * 64 + 32), r[1]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(tempty_bar)) : "memory");
            ok = store_boxes<kStoreSlots, AMAX>(&tmD, p.n_owners ? om.m : nullptr, store_area, boxgo_bar, r, ew, local, tn * kBN + cq * 64, tm * kBM + q * 32,
                                          p, alpha, abort_flag, am_plain, am_rht);
        }
        if (AMAX) amax_flush(p, am_plain, am_rht);
        if (lane == 0) bulk_wait_all();   // this lane's stores are in global memory before the CTA exits
    } else {
        // ------------------------------- scale warps (18..21) -------------------------------
        // Per stage, each warp writes the stage's block scales into its 32 TMEM lanes in the
        // layout the block-scaled MMA reads: for 64-wide K step j, the scales of A sit in columns
        // 4j..4j+3 of the stage's A region and lane i of every quadrant holds the 16-byte line i
        // of the 512-byte scale tile (rows i, i+32, i+64, i+96); B's two 128-row tiles fill
        // columns 8j..8j+3 and 8j+4..8j+7 of the B region the same way.
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        int g = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
            for (int kb = 0; kb < p.num_kb; ++kb, ++g) {
                const int s = g % kStages;
                const uint32_t ph = (uint32_t)(g / kStages) & 1u;
                const bool landed = mbar_wait(smem_u32(&full_bar[s]), ph, abort_flag, p.flags, p.budget_ns);
                if (!__all_sync(0xFFFFFFFFu, landed)) {
                    ok = false;
                    break;
                }
                const uint8_t* sfa_s = smem + s * kStageBytes + kABytes + kBBytes;
                const uint8_t* sfb_s = sfa_s + kSFABytes;
                uint32_t ra[16], rb[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 a = *reinterpret_cast<const uint4*>(sfa_s + 512 * j + 16 * lane);
                    const uint4 b0 = *reinterpret_cast<const uint4*>(sfb_s + 512 * j + 16 * lane);
                    const uint4 b1 = *reinterpret_cast<const uint4*>(sfb_s + 2048 + 512 * j + 16 * lane);
                    ra[4 * j] = a.x; ra[4 * j + 1] = a.y; ra[4 * j + 2] = a.z; ra[4 * j + 3] = a.w;
                    rb[8 * j] = b0.x; rb[8 * j + 1] = b0.y; rb[8 * j + 2] = b0.z; rb[8 * j + 3] = b0.w;
                    rb[8 * j + 4] = b1.x; rb[8 * j + 5] = b1.y; rb[8 * j + 6] = b1.z; rb[8 * j + 7] = b1.w;
                }
                const uint32_t t_sfa = tmem + lane_base + kSfCol0 + s * kSfColsPerStage;
                tmem_st16(t_sfa, ra);
                tmem_st32(t_sfa + 16, rb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&sfready_bar[s])) : "memory");
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ---------------------------------------------------------------------------------------
// 2-SM variant: a cluster of two CTAs on an SM pair computes 256 x 256 output tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64).  CTA r of the pair holds rows
// [128 r, 128 r + 128) of the A tile and rows [128 r, 128 r + 128) of the B tile, and owns the
// 128 x 256 accumulator of its A rows.  Per 256-wide K block each SM loads 32 KiB of codes
// (the 1-SM tile loads 48 KiB), so five stages (with the scales) fit in shared memory.  Each
// CTA's block scales (A: its own 128 rows; B: all 256 rows) are 2D TMA boxes of 8-byte elements
// (one 128-row tile's 4 K steps = 2 KiB per box row).  All of a stage's loads, in both CTAs,
// complete on the leader's full barrier.  The leader CTA (rank 0) then moves the scales into
// TMEM with tcgen05.cp.cta_group::2 (each CTA from its own shared memory; in a cta_group::2
// kernel tcgen05.st from scale warps waits for the pair's queued MMAs, ~1400 cycles a stage)
// and issues the MMAs; its commits arrive in both CTAs.  Every copy is issued by the CTA that
// owns its destination.
// ---------------------------------------------------------------------------------------
constexpr int k2Stages = 5;
constexpr int k2ABytes = 128 * kBK / 2;                // 16384: this CTA's 128 A rows
constexpr int k2BBytes = 128 * kBK / 2;                // 16384: this CTA's half of the B tile
constexpr int k2CodeBytes = k2ABytes + k2BBytes;       // 32768: counted on the leader's full barrier
constexpr int k2StageBytes = k2CodeBytes + kSFABytes + kSFBBytes;  // + own A scales + all B scales = 38912
constexpr int k2SfRing = k2Stages;                     // one TMEM scale region per stage
constexpr int k2Threads = 576;                         // producer, MMA, 16 epilogue warps
constexpr int k2StoreSlots = 8;
constexpr int k2Smem = k2Stages * k2StageBytes + k2StoreSlots * kStoreSlotBytes + kBarrierBytes + 1024;
static_assert(k2Smem <= 232448, "SM-pair kernel shared memory");
constexpr uint32_t k2Idesc = (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
static_assert(kSfCol0 + k2SfRing * kSfColsPerStage <= kTmemCols, "TMEM budget (2-SM)");
static_assert(k2StageBytes % 1024 == 0, "stages keep 1024-byte alignment");

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the object at `saddr` (a shared::cta address) in CTA `rank`
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// arrive on an mbarrier of the other CTA of the pair.  The default (.release at .cta scope) form:
// what crosses the pair here is the completion of tcgen05 work, ordered by the tcgen05 fences
// around the thread synchronisation, and the .release.cluster form costs ~1100 cycles (measured).
__device__ __forceinline__ void arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, volatile uint32_t* abort, uint32_t* flags,
                                             uint64_t budget_ns, bool honor_abort = true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
        if (mbar_try_wait_cl(bar, parity)) return true;
    const uint64_t t0 = cycles(), limit = 2 * budget_ns;
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait_cl(bar, parity)) return true;
        if (honor_abort && *abort) return false;
        if (cycles() - t0 > limit) {
            *abort = 1u;
            atomicOr(flags, kFlagTimeout);
            return false;
        }
    }
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// arrive on the barrier at this shared::cta offset in both CTAs of the pair, when this thread's
// prior tcgen05 operations complete
__device__ __forceinline__ void mma_mxf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}
__device__ __forceinline__ void mma_commit_local_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// shared-memory descriptor of a 512-byte scale tile read by tcgen05.cp 32x128b: no swizzle, the
// 32 16-byte rows one after another (8-row core matrices 128 bytes apart)
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
           (1ull << 46);
}
// one 512-byte scale tile (32 rows x 16 bytes) into 4 TMEM columns of all four lane quadrants,
// in both CTAs of the pair, each from its own shared memory
__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}
// cancel `bytes` of a barrier phase's expected transaction count (copies that were never issued)
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// bytes of one stage's copies into one CTA: A and B rows, A's scale tiles, both B row tiles' scales
template <int F>
constexpr uint32_t k2StageTx = (uint32_t)(k2CodeBytes + 3 * OpFmt<F>::kTilesPerBlock * 512);
static_assert(k2StageTx<kNVF4> == (uint32_t)k2StageBytes, "NVFP4 stage fills its slot");

// kind::f16 instruction descriptor: fp32 accumulator (bits 4-5 = 1), A and B bf16 (bits 7-9 and
// 10-12 = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24
constexpr uint32_t k2IdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int F, bool AMAX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(k2Threads, 1)
    gemm_nvf4_2sm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                         const __grid_constant__ CUtensorMap tmD, const __grid_constant__ OwnerMaps om, GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* store_area = smem + k2Stages * k2StageBytes;
    uint8_t* bar_area = store_area + k2StoreSlots * kStoreSlotBytes;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(bar_area);          // leader: TMA bytes of both CTAs
    uint64_t* empty_bar = full_bar + k2Stages;                            // both: MMAs of the stage done
    uint64_t* tfull_bar = empty_bar + k2Stages;                           // both: accumulator ready
    uint64_t* tempty_bar = tfull_bar + 1;                                 // leader: both epilogues drained
    uint64_t* done_bar = tempty_bar + 1;
    uint64_t* boxgo_bar = done_bar + 1;                                   // store slot hand-over (store_boxes)
    uint64_t* edrained_bar = boxgo_bar + 2 * kEpi1Warps;                  // peer: its epilogue drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(edrained_bar + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    uint32_t* issued_slot = tmem_slot + 2;                                // stages this CTA's producer issued

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int ntiles = p.tiles_m * p.tiles_n;   // tiles_m counts 256-row tiles here

    if (threadIdx.x == 0) {
        for (int s = 0; s < k2Stages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        mbar_init(smem_u32(tfull_bar), 1);
        // the leader's epilogue warps arrive on it locally, the peer's drain as one forwarded arrival
        mbar_init(smem_u32(tempty_bar), kEpi1Warps + 1);
        mbar_init(smem_u32(edrained_bar), kEpi1Warps);
        mbar_init(smem_u32(done_bar), 1);
        for (int b = 0; b < 2 * kEpi1Warps; ++b) mbar_init(smem_u32(&boxgo_bar[b]), 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();   // barriers of both CTAs initialised, TMEM allocated in both
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------- producer (both CTAs) --------------------------------
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmSA)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmSB)) : "memory");
            int g = 0;
            bool ok = true;
            for (int t = pair; ok && t < ntiles; t += npairs) {
                int tm, tn;
                tile_coords(t, p, tm, tn);
                const int m0 = tm * 256 + (int)rank * 128, n0 = tn * kBN + (int)rank * 128;
                for (int kb = 0; kb < p.num_kb; ++kb, ++g) {
                    const int s = g % k2Stages;
                    const uint32_t ph = (uint32_t)(g / k2Stages) & 1u;
                    if (!mbar_wait_cl(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag, p.flags, p.budget_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = map_rank(smem_u32(&full_bar[s]), 0);
                    if (rank == 0) mbar_expect_tx(smem_u32(&full_bar[s]), 2u * k2StageTx<F>);
                    uint8_t* st = smem + s * k2StageBytes;
                    tma_load_2d_pair(smem_u32(st), &tmA, kb * 128, m0, full_leader);
                    tma_load_2d_pair(smem_u32(st + k2ABytes), &tmB, kb * 128, n0, full_leader);
                    // scales: this CTA's A row tile and both B row tiles of the pair tile, 4 K steps
                    // (2 KiB) per row tile; rows and K steps past the tensor read as zero
                    if (F != kBF16) {
                        constexpr int sfe = OpFmt<F>::kTilesPerBlock * 64;   // 8-byte elements per row tile per stage
                        tma_load_2d_pair(smem_u32(st + k2CodeBytes), &tmSA, kb * sfe, tm * 2 + (int)rank, full_leader);
                        tma_load_2d_pair(smem_u32(st + k2CodeBytes + kSFABytes), &tmSB, kb * sfe, tn * 2, full_leader);
                    }
                }
            }
            *issued_slot = (uint32_t)g;   // read by the leader's drain after the first cluster barrier
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer (leader only) ----------------------------
        // As in the 1-SM kernel the whole warp runs the loop and one elected lane issues.
        if (rank == 0) {
            const uint32_t sbase = smem_u32(smem);
            const uint64_t adesc0 = desc_k_sw128(sbase), bdesc0 = desc_k_sw128(sbase + k2ABytes);
            int g = 0, local = 0;
            bool ok = true;
            for (int t = pair; ok && t < ntiles; t += npairs, ++local) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_cl(smem_u32(tempty_bar), ((uint32_t)local & 1u) ^ 1u, abort_flag,
                                                          p.flags, p.budget_ns)))
                    break;
                tc_fence_after();
                for (int kb = 0; kb < p.num_kb; ++kb, ++g) {
                    const int s = g % k2Stages, f = g % k2SfRing;
                    const bool landed =
                        mbar_wait_cl(smem_u32(&full_bar[s]), (uint32_t)(g / k2Stages) & 1u, abort_flag, p.flags, p.budget_ns);
                    if (!__all_sync(0xFFFFFFFFu, landed)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    constexpr int tpb = OpFmt<F>::kTilesPerBlock;
                    const int steps = min(4, p.kst - 4 * kb);
                    const int tiles = min(tpb, p.nkt - tpb * kb);
                    const uint64_t aoff = (uint64_t)((s * k2StageBytes) >> 4);
                    const uint32_t t_sfa = tmem + kSfCol0 + f * kSfColsPerStage;
                    if (elect_one()) {
                        const uint32_t sf_s = sbase + s * k2StageBytes + k2CodeBytes;
#pragma unroll
                        for (int t = 0; t < tpb; ++t)
                            if (t < tiles) {
                                tmem_cp_sf_pair(t_sfa + 4 * t, desc_sf(sf_s + 512 * t));
                                tmem_cp_sf_pair(t_sfa + 16 + 8 * t, desc_sf(sf_s + kSFABytes + 512 * t));
                                tmem_cp_sf_pair(t_sfa + 20 + 8 * t, desc_sf(sf_s + kSFABytes + tpb * 512 + 512 * t));
                            }
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            if (j < steps) {
                                const int tj = OpFmt<F>::tile_of_step(j);
                                if (F == kMXF4)
                                    mma_mxf4_pair(tmem, adesc0 + aoff + 2 * j, bdesc0 + aoff + 2 * j,
                                                  OpFmt<F>::idesc(k2Idesc, j), t_sfa + 4 * tj, t_sfa + 16 + 8 * tj,
                                                  (kb | j) != 0 ? 1u : 0u);
                                else if (F == kBF16)
                                    mma_bf16_pair(tmem, adesc0 + aoff + 2 * j, bdesc0 + aoff + 2 * j, k2IdescBf16,
                                                  (kb | j) != 0 ? 1u : 0u);
                                else
                                    mma_nvf4_pair(tmem, adesc0 + aoff + 2 * j, bdesc0 + aoff + 2 * j, k2Idesc, t_sfa + 4 * tj,
                                                  t_sfa + 16 + 8 * tj, (kb | j) != 0 ? 1u : 0u);
                            }
                        mma_commit_pair(smem_u32(&empty_bar[s]));
                    }
                    __syncwarp();
                }
                if (ok && elect_one()) mma_commit_pair(smem_u32(tfull_bar));
                __syncwarp();
            }
            if (elect_one()) mma_commit_local_pair(smem_u32(done_bar));
            __syncwarp();
            mbar_wait_cl(smem_u32(done_bar), 0u, abort_flag, p.flags, kDrainBudgetNs, false);
        } else {
            // The peer's MMA warp forwards its CTA's drained accumulator to the leader as one
            // remote arrival per tile, so the epilogue warps arrive locally (cheap) and one remote
            // arrival crosses the pair.
            const uint32_t tempty_leader = map_rank(smem_u32(tempty_bar), 0);
            int local = 0;
            for (int t = pair; t < ntiles; t += npairs, ++local) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(edrained_bar), (uint32_t)local & 1u, abort_flag, p.flags,
                                                       p.budget_ns)))
                    break;
                if (lane == 0) arrive_cluster(tempty_leader);
                __syncwarp();
            }
        }
    } else if (warp < 2 + kEpi1Warps) {
        // ------------------------------- epilogue (both CTAs) --------------------------------
        // As in the 1-SM kernel: 16 warps x 64 columns of this CTA's 128 accumulator rows, TMEM
        // released before the TMA stores: on the leader's barrier directly (leader CTA) or through
        // the peer's forwarding warp.
        const int ew = warp - 2;
        const int q = warp & 3;
        const int cq = ew >> 2;
        const float alpha = p.sta ? __fmul_rn(*p.sta, *p.stb) : 1.0f;   // MXFP4: no tensor scales
        const uint32_t drained = smem_u32(rank == 0 ? tempty_bar : edrained_bar);
        int local = 0;
        bool ok = true;
        uint32_t am_plain = 0;
        float am_rht = 0.0f;
        for (int t = pair; ok && t < ntiles; t += npairs, ++local) {
            int tm, tn;
            tile_coords(t, p, tm, tn);
            const bool full = mbar_wait_cl(smem_u32(tfull_bar), (uint32_t)local & 1u, abort_flag, p.flags, p.budget_ns);
            if (!__all_sync(0xFFFFFFFFu, full)) break;
            tc_fence_after();
            uint32_t r[2][32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cq * 64), r[0]);
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cq * 64 + 32), r[1]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(drained) : "memory");
            ok = store_boxes<k2StoreSlots, AMAX>(&tmD, p.n_owners ? om.m : nullptr, store_area, boxgo_bar, r, ew, local, tn * kBN + cq * 64,
                                           tm * 256 + (int)rank * 128 + q * 32, p, alpha, abort_flag, am_plain, am_rht);
        }
        if (AMAX) amax_flush(p, am_plain, am_rht);
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    cluster_sync_all();   // both producers have stopped issuing and published their stage counts
    if (warp == 0 && lane == 0 && rank == 0) {
        // Drain: every copy of either CTA lands before either exits.  All copies of a stage land on
        // the leader's full barrier, so the leader waits there for the stages that may still be
        // outstanding.  A producer cannot run more than k2Stages ahead of the slower one (a slot is
        // refilled only after the MMAs consumed it, which needs both CTAs' copies), so those are
        // the last k2Stages before the larger count, one phase per barrier.  After an abort the
        // two counts can differ: a stage only the peer issued has its missing arrival made here
        // (for the peer's bytes); a stage only the leader issued has the peer's bytes cancelled.
        // After a normal run both counts are equal, all stages were consumed, and every wait
        // returns at once.
        const int gl = (int)*issued_slot;
        const int gp = (int)ld_cluster_u32(map_rank(smem_u32(issued_slot), 1));
        const int gmax = max(gl, gp);
        for (int k = max(0, gmax - k2Stages); k < gmax; ++k) {
            const uint32_t bar = smem_u32(&full_bar[k % k2Stages]);
            if (k >= gl)
                mbar_expect_tx(bar, k2StageTx<F>);
            else if (k >= gp)
                mbar_complete_tx(bar, k2StageTx<F>);
            mbar_wait_cl(bar, (uint32_t)(k / k2Stages) & 1u, abort_flag, p.flags, kDrainBudgetNs, false);
        }
    }
    cluster_sync_all();   // both CTAs finished with TMEM, barriers and each other's shared memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// 2D map over codes [rows][k/2] bytes, box = 128 bytes x box_rows, 128-byte swizzle, zero fill
static bool make_code_map(CUtensorMap* map, const void* codes, int64_t rows, int64_t k, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
    cuuint32_t box[2] = {128u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2D map over the swizzled scale tiles of a form, in 8-byte elements: row = 128-row tile,
// nkt x 512 bytes per row; box = the scale tiles of one 256-wide K block (4 for NVFP4, 2 for MXFP4,
// 64 elements each) x box_rows
static bool make_sf_map(CUtensorMap* map, const void* scales, int64_t row_tiles, int64_t nkt, uint32_t box_rows,
                        uint32_t box_elems) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(nkt * 64), (cuuint64_t)row_tiles};
    cuuint64_t strides[1] = {(cuuint64_t)(nkt * 512)};
    cuuint32_t box[2] = {box_elems, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(scales), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2D map over the output D[M][ldd] (bf16 or fp32), box = 128 bytes x 32 rows, 128-byte swizzle;
// rows >= M and columns >= N of a box are not written
static bool make_out_map(CUtensorMap* map, void* d, int64_t M, int64_t N, int64_t ldd, bool fp32) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int64_t esz = fp32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(ldd * esz)};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, d, dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The dynamic shared-memory limit is a per-device attribute of a kernel: raise it once on each
// device (bit d of `done`) before the first launch there.
static cudaError_t ensure_smem_attr(const void* kernel, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// SM count of the current device, looked up once per device
static int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Output maps of the reduce-scatter epilogue: owner o's shard holds rows
// [o * owner_rows, min(M, (o + 1) * owner_rows)) of D, fp32, row stride ldd
static bool make_owner_maps(OwnerMaps* om, float* const* shards, int n_owners, int64_t owner_rows, int64_t M, int64_t N,
                            int64_t ldd) {
    *om = OwnerMaps{};
    for (int o = 0; o < n_owners; ++o) {
        const int64_t rows = std::min(owner_rows, M - o * owner_rows);
        if (rows < 1 || !make_out_map(&om->m[o], shards[o], rows, N, ldd, true)) return false;
    }
    return true;
}

// n_owners > 0: the reduce-scatter epilogue (fp32 adds into owner_d[o]) replaces the stores to d
template <bool MX>
static cudaError_t launch_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_st, int64_t M,
                               const uint8_t* b_codes, const uint8_t* b_scales, const float* b_st, int64_t N, int64_t K,
                               void* d, int64_t ldd, bool out_fp32, uint32_t* flags, uint64_t budget_ns,
                               cudaStream_t stream, float* const* owner_d = nullptr, int n_owners = 0,
                               int64_t owner_rows = 0, uint32_t* amax_out = nullptr, uint32_t rht_signs = 0) {
    if (amax_out && (out_fp32 || n_owners > 0 || M % 16 != 0)) return cudaErrorInvalidValue;
    if (n_owners < 0 || n_owners > kMaxOwners || (n_owners > 0 && (!out_fp32 || owner_rows < 32 || owner_rows % 32 != 0 ||
                                                                   (M + owner_rows - 1) / owner_rows != n_owners)))
        return cudaErrorInvalidValue;
    static const OwnerMaps no_owners{};
    OwnerMaps om_local;
    const OwnerMaps* om = &no_owners;
    if (n_owners > 0) {
        if (!make_owner_maps(&om_local, owner_d, n_owners, owner_rows, M, N, ldd)) return cudaErrorInvalidValue;
        om = &om_local;
        d = owner_d[0];   // the plain output map is built but never written
    }
    GemmParams p{};   // value-initialized: every field not set below is zero (no owners, no amax)
    p.sfa = a_scales;
    p.sfb = b_scales;
    p.sta = a_st;
    p.stb = b_st;
    p.d = d;
    p.ldd = ldd;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.M = (int32_t)M;
    p.N = (int32_t)N;
    p.K = (int32_t)K;
    p.nkt = (int32_t)(MX ? (K + 127) / 128 : (K + 63) / 64);
    p.kst = (int32_t)((K + 63) / 64);
    p.num_kb = (int32_t)((K + kBK - 1) / kBK);
    p.sfb_row_tiles = (int32_t)((N + 127) / 128);
    p.sfa_row_tiles = (int32_t)((M + 127) / 128);
    p.tiles_m = (int32_t)((M + kBM - 1) / kBM);
    p.tiles_n = (int32_t)((N + kBN - 1) / kBN);
    p.group_n = (M <= N) ? 1 : 0;   // operands are M x K and N x K: sweep the smaller one
    p.flags = flags;
    p.budget_ns = budget_ns;
    p.n_owners = n_owners;
    p.owner_rows = (int32_t)owner_rows;
    p.amax_out = amax_out;
    for (int i = 0; i < 16; ++i) p.rht_mask[i] = ((rht_signs >> i) & 1u) ? 0x80008000u : 0u;
    const int sms = sm_count();
    // SM-pair tiles for M >= 256 (fewer operand bytes per SM per K block, a deeper ring);
    // NVFP4_GEMM_VARIANT=1sm selects the 1-SM kernel for every shape (read on every call)
    const char* variant = getenv("NVFP4_GEMM_VARIANT");
    const bool force_1sm = variant && strcmp(variant, "1sm") == 0;
    if (!force_1sm && M >= 256 && sms >= 2) {
        static std::atomic<uint64_t> attr_2sm{0};
        auto kern2 = amax_out ? gemm_nvf4_2sm_kernel<MX ? kMXF4 : kNVF4, true> : gemm_nvf4_2sm_kernel<MX ? kMXF4 : kNVF4, false>;
        static std::atomic<uint64_t> attr_2sm_amax{0};
        if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern2), k2Smem, amax_out ? attr_2sm_amax : attr_2sm))
            return e;
        CUtensorMap ta2, tb2;
        if (!make_code_map(&ta2, a_codes, M, K, 128) || !make_code_map(&tb2, b_codes, N, K, 128)) return cudaErrorInvalidValue;
        p.tiles_m = (int32_t)((M + 255) / 256);
        const int64_t ntiles = (int64_t)p.tiles_m * p.tiles_n;
        const int64_t pairs = ntiles < sms / 2 ? ntiles : sms / 2;
        CUtensorMap td2, tsa, tsb;
        const uint32_t sfe = (uint32_t)OpFmt<MX ? kMXF4 : kNVF4>::kTilesPerBlock * 64u;
        if (!make_out_map(&td2, d, M, N, ldd, out_fp32) || !make_sf_map(&tsa, a_scales, p.sfa_row_tiles, p.nkt, 1, sfe) ||
            !make_sf_map(&tsb, b_scales, p.sfb_row_tiles, p.nkt, 2, sfe))
            return cudaErrorInvalidValue;
        kern2<<<(unsigned)(2 * pairs), k2Threads, k2Smem, stream>>>(ta2, tb2, tsa, tsb, td2, *om, p);
        return cudaGetLastError();
    }
    static std::atomic<uint64_t> attr_1sm{0};
    auto kern1 = amax_out ? gemm_nvf4_kernel<MX, true> : gemm_nvf4_kernel<MX, false>;
    static std::atomic<uint64_t> attr_1sm_amax{0};
    if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern1), kGemmSmem, amax_out ? attr_1sm_amax : attr_1sm))
        return e;
    CUtensorMap ta, tb;
    if (!make_code_map(&ta, a_codes, M, K, kBM) || !make_code_map(&tb, b_codes, N, K, kBN))
        return cudaErrorInvalidValue;
    const int64_t ntiles = (int64_t)p.tiles_m * p.tiles_n;
    const int grid = (int)(ntiles < sms ? ntiles : sms);
    CUtensorMap td;
    if (!make_out_map(&td, d, M, N, ldd, out_fp32)) return cudaErrorInvalidValue;
    kern1<<<grid, kGemm1Threads, kGemmSmem, stream>>>(ta, tb, td, *om, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm_nvf4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_st, int64_t M,
                             const uint8_t* b_codes, const uint8_t* b_scales, const float* b_st, int64_t N, int64_t K,
                             void* d, int64_t ldd, bool out_fp32, uint32_t* flags, uint64_t budget_ns,
                             cudaStream_t stream) {
    return launch_gemm<false>(a_codes, a_scales, a_st, M, b_codes, b_scales, b_st, N, K, d, ldd, out_fp32, flags,
                              budget_ns, stream);
}

cudaError_t launch_gemm_nvf4_reduce_scatter(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_st, int64_t M,
                                            const uint8_t* b_codes, const uint8_t* b_scales, const float* b_st, int64_t N,
                                            int64_t K, float* const* shards, int n_owners, int64_t owner_rows, int64_t ldd,
                                            uint32_t* flags, uint64_t budget_ns, cudaStream_t stream) {
    return launch_gemm<false>(a_codes, a_scales, a_st, M, b_codes, b_scales, b_st, N, K, nullptr, ldd, true, flags,
                              budget_ns, stream, shards, n_owners, owner_rows);
}

cudaError_t launch_gemm_nvf4_amax(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_st, int64_t M,
                                  const uint8_t* b_codes, const uint8_t* b_scales, const float* b_st, int64_t N, int64_t K,
                                  void* d, int64_t ldd, uint32_t* amax_out, uint32_t rht_signs, uint32_t* flags,
                                  uint64_t budget_ns, cudaStream_t stream) {
    return launch_gemm<false>(a_codes, a_scales, a_st, M, b_codes, b_scales, b_st, N, K, d, ldd, false, flags, budget_ns,
                              stream, nullptr, 0, 0, amax_out, rht_signs);
}

// MXFP4 operands carry no tensor scale (null scale pointers: the epilogue's factor is 1)
cudaError_t launch_gemm_mxf4(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M, const uint8_t* b_codes,
                             const uint8_t* b_scales, int64_t N, int64_t K, void* d, int64_t ldd, bool out_fp32,
                             uint32_t* flags, uint64_t budget_ns, cudaStream_t stream) {
    return launch_gemm<true>(a_codes, a_scales, nullptr, M, b_codes, b_scales, nullptr, N, K, d, ldd, out_fp32, flags,
                             budget_ns, stream);
}

// 2D map over a bf16 operand [rows][ld] viewed as bytes: box = 128 bytes (64 elements) x 128 rows,
// 128-byte swizzle, zero fill past the tensor (the same smem layout as a stage of FP4 codes)
static bool make_bf16_map(CUtensorMap* map, const void* p, int64_t rows, int64_t K, int64_t ld) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K * 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {128u, 128u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(p), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// D[M][N] = A[M][K] . B[N][K]^T in bf16 with fp32 accumulation, on the SM-pair kernel (every M:
// rows past M read as zero and are not stored)
cudaError_t launch_gemm_bf16(const uint16_t* a, int64_t lda, const uint16_t* b, int64_t ldb, int64_t M, int64_t N,
                             int64_t K, void* d, int64_t ldd, bool out_fp32, uint32_t* flags, uint64_t budget_ns,
                             cudaStream_t stream) {
    static std::atomic<uint64_t> attr{0};
    if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(gemm_nvf4_2sm_kernel<kBF16, false>), k2Smem, attr))
        return e;
    GemmParams p{};   // value-initialized: every field not set below is zero (no owners, no amax)
    std::memset(&p, 0, sizeof(p));
    p.d = d;
    p.ldd = ldd;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.M = (int32_t)M;
    p.N = (int32_t)N;
    p.K = (int32_t)K;
    p.nkt = 0;
    p.kst = (int32_t)((2 * K + 31) / 32);       // 32 bytes (16 elements) per MMA
    p.num_kb = (int32_t)((2 * K + 127) / 128);  // 128 bytes (64 elements) per stage
    p.sfb_row_tiles = (int32_t)((N + 127) / 128);
    p.sfa_row_tiles = (int32_t)((M + 127) / 128);
    p.tiles_m = (int32_t)((M + 255) / 256);
    p.tiles_n = (int32_t)((N + kBN - 1) / kBN);
    p.group_n = (M <= N) ? 1 : 0;
    p.flags = flags;
    p.budget_ns = budget_ns;
    const int sms = sm_count();
    CUtensorMap ta, tb, td;
    if (!make_bf16_map(&ta, a, M, K, lda) || !make_bf16_map(&tb, b, N, K, ldb) || !make_out_map(&td, d, M, N, ldd, out_fp32))
        return cudaErrorInvalidValue;
    const int64_t ntiles = (int64_t)p.tiles_m * p.tiles_n;
    const int64_t pairs = ntiles < sms / 2 ? ntiles : sms / 2;
    // the scale maps are not read by the bf16 instantiation; valid maps are passed in their place
    static const OwnerMaps no_owners{};
    gemm_nvf4_2sm_kernel<kBF16, false><<<(unsigned)(2 * pairs), k2Threads, k2Smem, stream>>>(ta, tb, ta, tb, td, no_owners, p);
    return cudaGetLastError();
}

}  // namespace nvfp4
