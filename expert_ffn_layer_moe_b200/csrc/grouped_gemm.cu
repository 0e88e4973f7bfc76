// grouped_gemm.cu -- ragged grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent kernel per GEMM of the expert FFN.  Each expert's rows form a
// group (MoE-latency article, section "router 之后还有一串动作": every expert runs
// its own matrix, and a grouped GEMM merges them into one launch; FinDEP review,
// section "核心公式": an expert is three GEMMs).  Two instantiations:
//   * SWIGLU = true : h[r] = bf16( silu(x W1[e]^T) * (x W3[e]^T) ).  A CTA's 128 weight
//                     rows are 64 rows of W1 and the same 64 rows of W3, so one
//                     accumulator holds g (TMEM lanes 0-63) and u (lanes 64-127), the
//                     activation tile is read once per K step, and the epilogue pairs
//                     the lanes through shared memory;
//   * SWIGLU = false: y[r] = h W2[e]^T, stored in fp32 (the combine sums k of these rows
//                     before the one rounding of the layer output).
//
// Tile shape ("swap-AB"): the MMA's M side walks the weight's output features, its N
// side (up to BN = 32..256 rows) walks the group's token rows.  Decode-sized groups (a
// few dozen rows per expert) then fill the tensor core's N side instead of padding M,
// and every weight byte is read once per token tile.  The MMA width is set per tile
// (the instruction descriptor is a runtime operand): a tile holding r rows multiplies
// round_up(r, 16) of them.
//
// CTA pairs (PAIR = true, the default): a cluster of two CTAs on two SMs shares one
// tcgen05.mma.cta_group::2 of M = 256.  CTA r holds weight rows [128 r, 128 r + 128) and
// half of the token tile; both CTAs' TMA loads complete on the leader's stage barrier,
// the leader issues the MMAs and its commits arrive at both CTAs' barriers, and each CTA
// drains its own TMEM.  An activation tile is then read once per 256 weight rows.  Tiny
// batches whose tiles would not cover the SM pairs use single-CTA tiles (PAIR = false).
//
// Warp roles (192 threads -- 480 with W8, below -- one CTA per SM, persistent over work items):
//   warp 0 lane 0 : TMA producer -- the 128-row weight tile and this CTA's part of the
//                   token tile per stage, 128-byte swizzle, mbarrier transaction counts;
//   warp 1        : TMEM allocator; lane 0 of the leader issues tcgen05.mma (bf16 in,
//                   fp32 accumulate) and tcgen05.commit to free stages and hand
//                   accumulators over;
//   warps 2..5    : epilogue -- tcgen05.ld of the accumulator (one TMEM lane quadrant
//                   per warp), staged through shared memory into 16-byte row stores.
// TMEM holds two accumulators of BN columns (W8: and four 32-column operand slots), so
// one tile's epilogue overlaps the next tile's main loop.  Barrier set-up and TMEM allocation run before the kernel waits on
// the previous kernel in the stream (programmatic dependent launch).
//
// fp8 weights (W8 = true; MoE-latency article, section "优化从测量开始": quantized
// weights as an experiment of their own): the weights are e4m3 bytes with one fp32 scale
// per output row.  The tensor cores take bf16 here, so the bytes are widened on chip:
//   warp 0        : TMA of 128 x 128-byte fp8 tiles (two 64-wide K blocks each);
//   warp 14       : TMA of the activation tiles (their own ring, as deep in K);
//   warps 6..13   : converters -- warp w widens the rows of TMEM lane quadrant w % 4,
//                   half (w - 6) / 4 of each K block, with integer operations and one
//                   exact bf16 multiplication, and stores them with tcgen05.st into one
//                   of four operand slots in TMEM;
//   warp 1        : MMA with A read from TMEM (tcgen05.mma [d], [a], b_desc);
//   epilogue      : as above, multiplying each output row by its scale first.
// W8 runs single-CTA tiles of up to 128 token rows (a pair's MMA would need the other
// CTA to signal every K step across the cluster, which costs more than the pair saves).
//
// fp8 weights and fp8 activations (A8 = true; the same section names activations beside
// weights): both operands are e4m3 bytes with one fp32 scale per row -- a weight row, or
// a token row of the activations.  The pipeline is the bf16 one (pairs included): a stage
// holds 128-byte rows, i.e. 128 K values instead of 64, and the MMA is
// tcgen05.mma.kind::f8f6f4 (K = 32 per instruction, fp32 accumulation of exact
// products), so each weight byte costs a quarter of the MMA instructions of the widened
// path.  The epilogue multiplies the accumulator by the weight row's scale and the token
// row's scale.
//
// Work items are (group, feature tile, K slice, token tile), enumerated on the device
// from the row offsets with no host synchronisation; empty groups produce no items (no
// padding to a fixed capacity).  The plain GEMM can split K into `ksplit` slices whose
// partial sums land in separate buffers `split_stride` apart, for shapes with too few
// tiles to cover the SMs; the consumer adds them in a fixed order, so results stay
// deterministic.  Every wait is bounded (globaltimer): on expiry the kernel records
// MOE_DEVERR_PIPELINE_TIMEOUT, lets in-flight copies drain, frees TMEM and returns.
#include <cmath>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;     // MMA M: weight rows per tile
constexpr int kBK = 64;      // K per pipeline stage: 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;   // K of one tcgen05.mma kind::f16
constexpr int kMaxGroups = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait, far above any legal wait

constexpr int pow2_at_least(int v, int p = 32) { return p >= v ? p : pow2_at_least(v, p * 2); }

template <int BN, bool SWIGLU, bool PAIR, bool W8, bool A8>
struct Cfg {
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "token tile must be 32..256, step 32");
    static_assert(!(W8 && A8), "fp8 activations use the native fp8 MMA, not the widening path");
    // K values per pipeline stage: one 128-byte row of the operand tiles (64 bf16 or 128 e4m3)
    static constexpr int kKStep = A8 ? 2 * kBK : kBK;
    // warps: producer, MMA, 4 epilogue; with W8 also 8 converter warps (fp8 -> bf16)
    // and an activation producer
    static_assert(!(W8 && PAIR), "fp8 weights run single-CTA tiles");
    static constexpr int kThreads = W8 ? 480 : 192;
    static constexpr int kCtas = PAIR ? 2 : 1;             // CTAs sharing one MMA (cta_group)
    static constexpr int kFeat = SWIGLU ? kBM / 2 : kBM;   // output features per CTA per tile
    static constexpr int kFeatTile = kCtas * kFeat;        // output features per work item
    static constexpr int kBRows = BN / kCtas;              // token rows of B held by each CTA
    static constexpr int kABytes = kBM * kBK * 2;          // 16 KB weight tile per stage
    static constexpr int kBBytes = kBRows * kBK * 2;
    // bf16: one TMA ring whose stages hold the weight and the activation tile.
    // W8: three rings -- fp8 weight tiles (deep: those loads go to HBM), activation
    // tiles (its stages are only kBBytes; the loads mostly hit L2) and the bf16 operand
    // slots the converter warps write for the MMA.
    static constexpr int kW8Bytes = W8 ? kBM * 2 * kBK : 0;  // one fp8 weight tile: K = 128 (16 KB)
    static constexpr int kABufs = W8 ? 4 : 0;              // bf16 operand slots in TMEM (two per fp8 tile)
    static constexpr int kACols = 32;                      // TMEM columns of one slot: 64 bf16 per lane
    static constexpr int kStageBytes = W8 ? kBBytes : kABytes + kBBytes;
    static constexpr int kStagesFit = (200 * 1024) / kStageBytes;
    // W8: the activation ring reaches as many K blocks ahead as the fp8 ring (two per
    // fp8 tile): both kinds of load take microseconds under full HBM traffic
    static constexpr int kFFit = W8 ? (200 * 1024) / (kW8Bytes + 2 * kBBytes) : 0;
    static constexpr int kFStages = kFFit > 8 ? 8 : kFFit;     // fp8 ring (W8)
    static constexpr int kStages = W8 ? 2 * kFStages : (kStagesFit > 10 ? 10 : kStagesFit);
    static constexpr int kAccCols = BN;                    // fp32 TMEM columns per accumulator
    static constexpr int kAccBufs = 2;
    static constexpr int kASlot0 = kAccBufs * kAccCols;    // W8: first TMEM column of the operand slots
    static constexpr int kTmemCols = pow2_at_least(kAccBufs * kAccCols + kABufs * kACols);
    static constexpr int kBarBytes = 8 * (2 * kStages + 2 * kAccBufs + 2 * kFStages + kABufs);
    static constexpr int kTableBytes = (4 * 3 * (kMaxGroups + 1) + 15) & ~15;  // starts, ends, item prefix
    // epilogue staging: one region of 34 x 32 fp32 per epilogue warp (a padded [32][33]
    // tile, or a dense [32][32] box for bulk stores at its 128-byte-aligned start); the
    // SwiGLU epilogue uses it as 2 x [64][33]
    static constexpr int kEpiWarpFloats = 34 * 32;
    static constexpr int kEpiBytes = 4 * kEpiWarpFloats * 4;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kFStages * kW8Bytes + kBarBytes + 16 +
                                      kTableBytes + kEpiBytes;
    // tcgen05 instruction descriptor: D=f32 (bit 4); kind::f16 with A=B=bf16 (format 1 at
    // bits 7 and 10), or kind::f8f6f4 with A=B=e4m3 (format 0); both operands K-major,
    // M>>4 at bit 24 (M = 128 per CTA, 256 per pair); N>>3 (bit 17) per tile.
    static constexpr uint32_t kIdescNoN = (1u << 4) | (A8 ? 0u : (1u << 7) | (1u << 10)) |
                                          ((uint32_t)((kBM * kCtas) >> 4) << 24);
    static_assert(kStages >= 2, "pipeline needs at least two stages");
    static_assert(!W8 || kFStages >= 2, "fp8 ring needs at least two tiles");
    static_assert(kTmemCols <= 512, "TMEM has 512 columns");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// ------------------------------------------------------------ PTX wrappers --
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity; false on timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) return false;
        }
    }
}

// Two e4m3 bytes, placed in bits 0-7 and 16-23 of `t`, -> two bf16 (low half first).
// t * 16 puts each byte's 7 exponent-and-mantissa bits at bits 4-10 of its half and
// its sign at bit 11; adding 15 times the sign bit carries it to bit 15 (2^11 + 15 *
// 2^11 = 2^15, no carry leaves the half).  The result is the bf16 whose value is the
// e4m3 value times 2^-120 -- exactly, since the e4m3 subnormals (exponent field 0)
// land on the bf16 subnormals with the same mantissa -- and one bf16 multiplication by
// 2^120 (exact: a power of two, no overflow) gives the value itself.
__device__ __forceinline__ uint32_t e4m3_pair_to_bf16x2(uint32_t t)
{
    const uint32_t a = t << 4;
    const uint32_t w = a + (a & 0x08000800u) * 15u;
    const __nv_bfloat162 two120 = __halves2bfloat162(__ushort_as_bfloat16((unsigned short)0x7B80),
                                                     __ushort_as_bfloat16((unsigned short)0x7B80));
    const __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&w), two120);
    return *reinterpret_cast<const uint32_t *>(&r);
}

// Four e4m3 bytes -> four bf16, as two words (bytes 0,1 and bytes 2,3).
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t v, uint32_t &lo, uint32_t &hi)
{
    lo = e4m3_pair_to_bf16x2(__byte_perm(v, 0u, 0x4140));  // byte 0 -> bits 0-7, byte 1 -> bits 16-23
    hi = e4m3_pair_to_bf16x2(__byte_perm(v, 0u, 0x4342));
}

// 16 consecutive 32-bit TMEM columns of this thread's lane (the warp's lane quadrant).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// 32 of the 128 fp8 values of row r of a 128 x 128 fp8 weight tile as TMA wrote it
// (128-byte rows, 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r & 7)):
// K block kh (0, 1), values [32 kq, 32 kq + 32) of its 64, as 16 bf16 pairs (low half =
// lower K), the layout of one lane of an MMA A operand in TMEM.
__device__ __forceinline__ void widen_e4m3_32(const uint8_t *src_tile, int r, int kh, int kq, uint32_t (&o)[16])
{
    const uint8_t *src = src_tile + r * 128;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = 4 * kh + 2 * kq + i;
        const uint4 v = *reinterpret_cast<const uint4 *>(src + ((c ^ (r & 7)) << 4));
        e4m3x4_to_bf16x4(v.x, o[8 * i + 0], o[8 * i + 1]);
        e4m3x4_to_bf16x4(v.y, o[8 * i + 2], o[8 * i + 3]);
        e4m3x4_to_bf16x4(v.z, o[8 * i + 4], o[8 * i + 5]);
        e4m3x4_to_bf16x4(v.w, o[8 * i + 6], o[8 * i + 7]);
    }
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap *m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with
// 128-byte swizzle: rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart (SBO),
// descriptor version 1 (bits 46..48), swizzle mode 2 = 128B (bits 61..63).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;              // leading byte offset: unused for swizzled K-major
    d |= (uint64_t)(1024 >> 4) << 32;    // stride byte offset
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// MMA with the A operand in TMEM (rows on lanes, K along the columns) and B in shared memory.
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (the warp's lane quadrant),
// without the wait: the registers are valid only after tmem_wait_ld on them (which
// names them as operands, so no use can be scheduled before it).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
          "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
          "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
          "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
}

// The load and its wait: 32 fp32 columns ready in registers.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    tmem_ld32_async(taddr, r);
    tmem_wait_ld(r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// One 32 x 32 fp32 box (32 output rows of 32 consecutive features) from this CTA's
// shared memory to global memory through the output map, as one bulk group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *m, int c0, int c1, uint32_t src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(src)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// ---------------------------------------------- CTA-pair (cta_group::2) forms --
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA loads into this CTA's shared memory that complete on `bar` (a shared::cluster
// address; with PAIR it may be the leader CTA's barrier).  Never multicast.
template <bool PAIR>
__device__ __forceinline__ void tma_3d(void *dst, const CUtensorMap *m, int c0, int c1, int c2, uint32_t bar)
{
    if (PAIR)
        asm volatile(
            "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
            : "memory");
}

// Four rows (r0..r3) of a 2-D map whose box is one row high, K columns [c0, c0 + 64),
// written as four consecutive 128-byte rows at dst with the map's swizzle: the
// activation rows of a token tile gathered straight from x.  Never multicast.
template <bool PAIR>
__device__ __forceinline__ void tma_gather4(void *dst, const CUtensorMap *m, int c0, int r0, int r1, int r2, int r3,
                                            uint32_t bar)
{
    if (PAIR)
        asm volatile(
            "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
            : "memory");
}

template <bool PAIR>
__device__ __forceinline__ void tma_2d(void *dst, const CUtensorMap *m, int c0, int c1, uint32_t bar)
{
    if (PAIR)
        asm volatile(
            "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar)
            : "memory");
}

// TMEM allocation: with PAIR one warp of each CTA of the pair takes part.
template <bool PAIR>
__device__ __forceinline__ void tmem_alloc_g(uint32_t *slot, uint32_t ncols)
{
    if (PAIR)
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                     "r"(ncols)
                     : "memory");
    else
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                     "r"(ncols)
                     : "memory");
}

template <bool PAIR>
__device__ __forceinline__ void tmem_relinquish_g()
{
    if (PAIR) asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    else asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

template <bool PAIR>
__device__ __forceinline__ void tmem_dealloc_g(uint32_t taddr, uint32_t ncols)
{
    if (PAIR)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
    else
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// One MMA: with PAIR, M = 256 across the pair (each CTA's 128 weight rows), N split
// between the CTAs' halves of the token tile; issued by the leader CTA only.  F8: both
// operands e4m3 (kind::f8f6f4, K = 32), else bf16 (kind::f16, K = 16).
template <bool PAIR, bool F8>
__device__ __forceinline__ void umma_g(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate)
{
    if (PAIR && F8)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    else if (PAIR)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    else if (F8)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        umma_bf16(d_tmem, adesc, bdesc, idesc, accumulate);
}

// Arrive on `bar` when the MMAs issued so far complete; with PAIR the arrival goes
// to the barrier at the same offset in both CTAs of the pair.
template <bool PAIR>
__device__ __forceinline__ void umma_commit_g(uint64_t *bar)
{
    if (PAIR) {
        const uint16_t both = 0x3;
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                smem_u32(bar)),
            "h"(both)
            : "memory");
    } else {
        umma_commit(bar);
    }
}

// silu(z) = z / (1 + e^-z) with the hardware exponential and reciprocal: about five
// instructions instead of about twenty-five for the IEEE forms (whose division also
// branches to a slow path).  Relative error a few 1e-6, far below the bf16 rounding of h
// that follows; e^-z overflowing to infinity gives the limit 0.  The SwiGLU epilogue
// issues almost all of the kernel's instructions on four warps, so at long token
// tiles this is what keeps it shorter than the main loop.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }


// Named barrier for the four epilogue warps (barrier 0 is __syncthreads).
__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// ------------------------------------------------------------------ kernel --
// PAIR = true runs as clusters of two CTAs on two SMs: CTA r of a pair holds weight
// rows [128 r, 128 r + 128) of the work item's 256 and token rows
// [n/2 r, n/2 r + n/2) of its n; the leader (r = 0) issues the M=256 MMAs, both CTAs'
// TMA loads complete on the leader's stage barrier, its commits reach both CTAs'
// barriers, and each CTA drains its own half of the accumulator.
//
// GATHER = true (bf16 SwiGLU GEMM only): the activation operand is not a permuted copy
// but x itself; row r of the groups reads x row gather_rows[r] (row_to_token), loaded
// by tile::gather4 TMA requests -- four rows each, issued by all 32 lanes of warp 0 --
// so the dispatch never writes x_perm.
template <int BN, bool SWIGLU, bool PAIR, bool W8, bool A8, bool GATHER>
__global__ void __launch_bounds__(Cfg<BN, SWIGLU, PAIR, W8, A8>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_wa, const __grid_constant__ CUtensorMap tm_wb,
                        const __grid_constant__ CUtensorMap tm_act, const int32_t *__restrict__ offsets,
                        int groups, int rows_single, int64_t R, int K, int Nout,
                        void *__restrict__ out, int ksplit, int64_t split_stride,
                        const float *__restrict__ scale_a, const float *__restrict__ scale_b,
                        const float *__restrict__ scale_act, int64_t ldo, const int32_t *__restrict__ gather_rows,
                        const __grid_constant__ CUtensorMap tm_out, int tma_store,
                        const int32_t *__restrict__ ends, int *dev_err)
{
    using C = Cfg<BN, SWIGLU, PAIR, W8, A8>;
    static_assert(!GATHER || (SWIGLU && !W8 && !A8), "gathered activation rows: bf16 SwiGLU GEMM only");
    static_assert(!GATHER || C::kBRows % 4 == 0, "gather4 loads rows in fours");
    constexpr int kThreads = C::kThreads;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);  // 1024-aligned for SW128

    uint8_t *stages = smem;                                     // TMA ring (W8: activations)
    uint8_t *fring = smem + C::kStages * C::kStageBytes;        // W8: fp8 weight tiles
    // epilogue staging, 1024-byte aligned (every stage and fp8 tile is a multiple of 1 KB)
    float *epi_stage = reinterpret_cast<float *>(fring + C::kFStages * C::kW8Bytes);
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(epi_stage) + C::kEpiBytes);
    uint64_t *empty_bar = full_bar + C::kStages;
    uint64_t *tfull_bar = empty_bar + C::kStages;
    uint64_t *tempty_bar = tfull_bar + C::kAccBufs;
    uint64_t *ffull_bar = tempty_bar + C::kAccBufs;             // W8: fp8 tile landed
    uint64_t *fempty_bar = ffull_bar + C::kFStages;             // W8: fp8 tile read by every converter warp
    uint64_t *afull_bar = fempty_bar + C::kFStages;             // W8: operand slot written by every converter warp
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(afull_bar + C::kABufs);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_ok = reinterpret_cast<volatile int *>(tmem_slot + 2);
    int *g_off = reinterpret_cast<int *>(tmem_slot + 4);  // [groups+1] row offsets
    int *g_tile = g_off + (kMaxGroups + 1);               // [groups+1] work-item prefix
    int *g_end = g_tile + (kMaxGroups + 1);               // [groups] end row of each group

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // work-list walker: one per pair
    const int nunits = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int n_feat = (Nout + C::kFeatTile - 1) / C::kFeatTile;
    const int KB = (K + C::kKStep - 1) / C::kKStep;  // pipeline stages along K

    // ---- barriers and TMEM: nothing here reads global memory, so it overlaps the tail
    // of the previous kernel in the stream (programmatic dependent launch)
    pdl_launch_dependents();
    if (tid == 0) {
        *abort_flag = 0;
        for (int s = 0; s < C::kStages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
        for (int b = 0; b < C::kAccBufs; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 4 * C::kCtas);  // every epilogue warp of the pair releases
        }
        if (W8) {
            for (int j = 0; j < C::kFStages; ++j) { mbar_init(&ffull_bar[j], 1); mbar_init(&fempty_bar[j], 8); }
            for (int a = 0; a < C::kABufs; ++a) mbar_init(&afull_bar[a], 8);  // every converter warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc_g<PAIR>(tmem_slot, C::kTmemCols);
        tmem_relinquish_g<PAIR>();
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();  // both CTAs' barriers exist before either signals the other
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // from here on the previous kernels' outputs are complete and visible

    // ---- work list: row offsets and the prefix of (token tiles x feature tiles x K slices) per group
    if (offsets == nullptr) {
        if (tid == 0) { g_off[0] = 0; g_off[1] = rows_single; g_end[0] = rows_single; }
    } else {
        // group g is rows [offsets[g], ends[g]) when ends is given, else [offsets[g], offsets[g+1])
        for (int i = tid; i <= groups; i += kThreads) g_off[i] = offsets[i];
        for (int i = tid; i < groups; i += kThreads) g_end[i] = ends ? ends[i] : offsets[i + 1];
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        bool bad = false;
        for (int base = 0; base < groups; base += 32) {
            const int gi = base + lane;
            int items = 0;
            if (gi < groups) {
                const int lo = g_off[gi], hi = g_end[gi];
                if (lo < 0 || hi < lo || (int64_t)hi > R) bad = true;
                else items = ((hi - lo + BN - 1) / BN) * n_feat * ksplit;
            }
            int v = items;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            if (gi < groups) g_tile[gi + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) g_tile[0] = 0;
        if (__any_sync(0xffffffffu, bad) && lane == 0 && rank == 0)
            set_device_error(dev_err, MOE_DEVERR_BAD_OFFSETS);
    }
    __syncthreads();
    const int total = g_tile[groups];  // units with no work skip every role loop below

    // item -> (group, feature tile, K slice, first row, end row of the group).  The
    // feature tile (and K slice) runs fastest: units running side by side share a token
    // tile, so a large group streams its activation rows from HBM once while its weights
    // (a few tens of MB per expert) stay in L2.
    auto decode = [&](int item, int &g, int &feat, int &ks, int &row0, int &row_end) {
        int lo = 0, hi = groups - 1;
        while (lo < hi) {  // largest g with g_tile[g] <= item (skips empty groups)
            const int mid = (lo + hi + 1) >> 1;
            if (g_tile[mid] <= item) lo = mid; else hi = mid - 1;
        }
        g = lo;
        const int local = item - g_tile[g];
        const int nfk = n_feat * ksplit;
        const int fk = local % nfk;
        feat = fk / ksplit;
        ks = fk % ksplit;
        row0 = g_off[g] + (local / nfk) * BN;
        row_end = g_end[g];
    };
    // W8: slices start and end on 128-wide K blocks (one fp8 load); a last half block
    // past K reads zeros from both tensor maps and adds nothing
    auto kslice = [&](int ks, int &kb0, int &kb1) {
        if (W8) {
            const int KB2 = (KB + 1) / 2;
            kb0 = 2 * (int)((int64_t)ks * KB2 / ksplit);
            kb1 = 2 * (int)((int64_t)(ks + 1) * KB2 / ksplit);
        } else {
            kb0 = (int)((int64_t)ks * KB / ksplit);
            kb1 = (int)((int64_t)(ks + 1) * KB / ksplit);
        }
    };
    // MMA width of a tile: its rows rounded up to the instruction's step of 16
    auto mma_width = [&](int row0, int row_end) { return min(BN, (min(BN, row_end - row0) + 15) & ~15); };

    bool failed = false;
    if (warp == 0 && (GATHER || lane == 0)) {
        // ------------------------------------------------------ TMA producer
        // (lane 0; with GATHER the whole warp, each lane gathering four activation rows)
        if (lane == 0) {
            tma_prefetch_map(&tm_wa);
            if (SWIGLU) tma_prefetch_map(&tm_wb);
            tma_prefetch_map(&tm_act);
        }
        // every load of the pair completes on the leader's stage barrier
        const uint32_t full0 = PAIR ? mapa_shared(smem_u32(&full_bar[0]), 0) : smem_u32(&full_bar[0]);
        int stage = 0;
        uint32_t phase = 0;
        for (int item = unit; W8 && item < total && !failed; item += nunits) {
            // fp8 weight tiles, as far ahead as the fp8 ring reaches
            int g, feat, ks, row0, row_end, kb0, kb1;
            decode(item, g, feat, ks, row0, row_end);
            kslice(ks, kb0, kb1);
            const int frow = feat * C::kFeatTile;
            for (int kb = kb0; kb < kb1; kb += 2) {
                if (!mbar_wait(&fempty_bar[stage], phase ^ 1u, abort_flag)) { failed = true; *abort_flag = 1; break; }
                uint8_t *dst = fring + stage * C::kW8Bytes;
                const uint32_t fb = smem_u32(&ffull_bar[stage]);
                mbar_arrive_expect_tx(&ffull_bar[stage], C::kW8Bytes);
                if (SWIGLU) {
                    tma_3d<false>(dst, &tm_wa, kb * kBK, frow, g, fb);
                    tma_3d<false>(dst + C::kW8Bytes / 2, &tm_wb, kb * kBK, frow, g, fb);
                } else {
                    tma_3d<false>(dst, &tm_wa, kb * kBK, frow, g, fb);
                }
                if (++stage == C::kFStages) { stage = 0; phase ^= 1u; }
            }
        }
        for (int item = unit; !W8 && item < total && !failed; item += nunits) {
            int g, feat, ks, row0, row_end, kb0, kb1;
            decode(item, g, feat, ks, row0, row_end);
            kslice(ks, kb0, kb1);
            const int frow = feat * C::kFeatTile + (int)rank * C::kFeat;        // first weight row (W1 / W)
            const int trow = row0 + (PAIR ? (int)rank * (mma_width(row0, row_end) >> 1) : 0);
            // GATHER: the x rows of this lane's four tile rows, fixed for the whole item.
            // Tile rows past R (a ragged last tile) read x row 0; like rows of the next
            // group, their products are never stored.
            const bool gl = GATHER && 4 * lane < C::kBRows;
            int xr[4] = {0, 0, 0, 0};
            if (gl) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int64_t r = (int64_t)trow + 4 * lane + i;
                    xr[i] = r < R ? gather_rows[r] : 0;
                }
            }
            for (int kb = kb0; kb < kb1; ++kb) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag);
                if (GATHER) ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) { failed = true; if (lane == 0) *abort_flag = 1; break; }
                uint8_t *st = stages + stage * C::kStageBytes;
                const uint32_t fb = full0 + 8u * stage;
                const int kc = kb * C::kKStep;  // K coordinate (elements; bytes for e4m3)
                if (lane == 0) {
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], C::kCtas * C::kStageBytes);
                    if (SWIGLU) {
                        // rows 0-63: W1 features [frow, +64); rows 64-127: the same features of W3
                        tma_3d<PAIR>(st, &tm_wa, kc, frow, g, fb);
                        tma_3d<PAIR>(st + C::kABytes / 2, &tm_wb, kc, frow, g, fb);
                    } else {
                        tma_3d<PAIR>(st, &tm_wa, kc, frow, g, fb);
                    }
                    if (!GATHER) tma_2d<PAIR>(st + C::kABytes, &tm_act, kc, trow, fb);
                }
                if (gl) tma_gather4<PAIR>(st + C::kABytes + lane * 512, &tm_act, kc, xr[0], xr[1], xr[2], xr[3], fb);
                if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ------------------------------------------------------ MMA issuer (leader CTA)
        int stage = 0, acc = 0, ab = 0;
        uint32_t phase = 0, aphase = 0, abphase = 0;
        for (int item = unit; item < total && !failed; item += nunits) {
            int g, feat, ks, row0, row_end, kb0, kb1;
            decode(item, g, feat, ks, row0, row_end);
            kslice(ks, kb0, kb1);
            const uint32_t idesc = C::kIdescNoN | ((uint32_t)(mma_width(row0, row_end) >> 3) << 17);
            if (!mbar_wait(&tempty_bar[acc], aphase ^ 1u, abort_flag)) { failed = true; *abort_flag = 1; break; }
            tc_fence_after();
            const uint32_t d0 = tmem_base + (uint32_t)(acc * C::kAccCols);
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { failed = true; *abort_flag = 1; break; }
                if (W8 && !mbar_wait(&afull_bar[ab], abphase, abort_flag)) { failed = true; *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t sst = smem_u32(stages + stage * C::kStageBytes);
                if (W8) {
                    // A = the converters' bf16 slot in TMEM (8 columns per K step of 16),
                    // B = the activation stage
                    const uint32_t ta = tmem_base + (uint32_t)(C::kASlot0 + ab * C::kACols);
                    const uint64_t db = sdesc_sw128(sst);
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                        const uint32_t accumulate = (kb != kb0 || kk != 0) ? 1u : 0u;
                        umma_bf16_ta(d0, ta + 8 * kk, db + 2 * kk, idesc, accumulate);
                    }
                } else {
                    const uint64_t da = sdesc_sw128(sst);
                    const uint64_t db = sdesc_sw128(sst + C::kABytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                        const uint32_t accumulate = (kb != kb0 || kk != 0) ? 1u : 0u;
                        // +32 bytes of K per step inside the 128-byte swizzled row (encoded >> 4):
                        // 16 bf16 or 32 e4m3 values, one MMA's K either way
                        umma_g<PAIR, A8>(d0, da + 2 * kk, db + 2 * kk, idesc, accumulate);
                    }
                }
                umma_commit_g<PAIR>(&empty_bar[stage]);  // stage free (in both CTAs) once read
                if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                if (W8) {
                    // the operand slot is free when this K block's MMAs complete, which the
                    // commit above already signals on the activation stage's barrier
                    if (++ab == C::kABufs) { ab = 0; abphase ^= 1u; }
                }
            }
            if (failed) break;
            umma_commit_g<PAIR>(&tfull_bar[acc]);        // accumulator complete (in both CTAs)
            if (++acc == C::kAccBufs) { acc = 0; aphase ^= 1u; }
        }
    } else if (warp >= 2 && warp < 6) {
        // ------------------------------------------------------ epilogue
        // Per 32-row chunk every warp loads its TMEM lane quadrant (one feature, or one
        // half of a SwiGLU pair, across 32 rows) into a padded shared tile; after the
        // epilogue barrier the tile is read back so each lane stores 16 bytes of
        // consecutive features of one row.
        const int q = warp & 3;   // TMEM lane quadrant this warp may read
        const int ew = warp - 2;  // 0..3
        // no 16-byte vector straddles a row end and every one is 16-byte aligned
        const bool vec_ok = (Nout & 7) == 0 && (ldo & 3) == 0 && (split_stride & 3) == 0;
        const uint32_t tempty_leader = PAIR ? mapa_shared(smem_u32(&tempty_bar[0]), 0) : 0u;
        int acc = 0;
        uint32_t aphase = 0;
        for (int item = unit; item < total; item += nunits) {
            int g, feat, ks, row0, row_end;
            decode(item, g, feat, ks, row0, row_end);
            bool ok = true;
            if (SWIGLU) {
                // one waiter decides for all four warps, so the named barriers of the
                // SwiGLU epilogue are always reached by all of them
                if (ew == 0 && lane == 0) *epi_ok = mbar_wait(&tfull_bar[acc], aphase, abort_flag) ? 1 : 0;
                epilogue_sync();
                ok = *epi_ok != 0;
                epilogue_sync();  // everyone has read the flag before it can be rewritten
            } else {
                // the plain epilogue has no barrier between its warps: each waits on its own
                if (lane == 0) ok = mbar_wait(&tfull_bar[acc], aphase, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            }
            if (!ok) { failed = true; if (lane == 0) *abort_flag = 1; break; }
            tc_fence_after();
            const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::kAccCols);
            const int nrows = min(BN, row_end - row0);
            if (SWIGLU) {
                float(*Gs)[33] = reinterpret_cast<float(*)[33]>(epi_stage);            // [64][33] g
                float(*Us)[33] = reinterpret_cast<float(*)[33]>(epi_stage + 64 * 33);  // [64][33] u
                float(*mine)[33] = q < 2 ? Gs : Us;
                const int fl = (q & 1) * 32 + lane;  // feature within this CTA's 64
                const int rr = lane >> 3, j = lane & 7;
                const int fv = feat * C::kFeatTile + (int)rank * C::kFeat + 8 * j;
                uint16_t *outh = static_cast<uint16_t *>(out);
                float sc = 1.0f;  // fp8 weights: the scale of this lane's weight row (W1 for g, W3 for u)
                if (W8 || A8) {
                    const int row = feat * C::kFeatTile + (int)rank * C::kFeat + fl;
                    sc = row < Nout ? (q < 2 ? scale_a : scale_b)[(int64_t)g * Nout + row] : 0.0f;
                }
                for (int c0 = 0; c0 < nrows; c0 += 32) {
                    float a[32];
                    tmem_ld32(t0 + c0, a);
                    // A8: column c is token row row0 + c0 + c, with its own scale (lane c holds it)
                    const float sa = A8 && c0 + lane < nrows ? scale_act[row0 + c0 + lane] : 0.0f;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        float v = (W8 || A8) ? a[c] * sc : a[c];
                        if (A8) v *= __shfl_sync(0xffffffffu, sa, c);
                        mine[fl][c] = v;
                    }
                    epilogue_sync();
                    // warp ew stores rows 8*ew .. 8*ew+7 of the chunk: 4 rows x 8 feature octets per step
#pragma unroll
                    for (int it = 0; it < 2; ++it) {
                        const int r = 8 * ew + 4 * it + rr;
                        if (c0 + r < nrows && fv < Nout) {
                            float h[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) h[i] = silu(Gs[8 * j + i][r]) * Us[8 * j + i][r];
                            uint4 v;
                            v.x = pack_bf16x2(h[0], h[1]);
                            v.y = pack_bf16x2(h[2], h[3]);
                            v.z = pack_bf16x2(h[4], h[5]);
                            v.w = pack_bf16x2(h[6], h[7]);
                            *reinterpret_cast<uint4 *>(outh + (size_t)(row0 + c0 + r) * Nout + fv) = v;
                        }
                    }
                    epilogue_sync();
                }
            } else {
                float *outf = static_cast<float *>(out) + (int64_t)ks * split_stride;
                const int fbase = feat * C::kFeatTile + (int)rank * C::kFeat + q * 32;
                const float sc =
                    (W8 || A8) ? (fbase + lane < Nout ? scale_a[(int64_t)g * Nout + fbase + lane] : 0.0f) : 1.0f;
                // The next chunk's TMEM load is in flight while this one is stored, and the
                // accumulator goes back to the MMA as soon as its last chunk is in registers.
                // With tma_store, a chunk of 32 whole rows leaves as one 32 x 32 fp32 box
                // from this warp's 4 KB staging tile (one bulk store issued by lane 0); a
                // ragged last chunk, and everything without tma_store, goes through the
                // padded tile: 8 16-byte stores per 32 rows instead of 32 4-byte ones (store
                // instruction issue, not bytes, limits short-K tiles).
                float *wreg = epi_stage + ew * C::kEpiWarpFloats;  // this warp's staging region
                float(*stage_t)[33] = reinterpret_cast<float(*)[33]>(wreg);
                float *box = wreg;  // [32 rows][32 features] (tma_store), 128-byte aligned
                const uint32_t box_s = smem_u32(box);
                static_assert((C::kEpiWarpFloats * 4) % 128 == 0, "bulk-store boxes start on 128 bytes");
                uint32_t cur[32], nxt[32];
                tmem_ld32_async(t0, cur);
                tmem_wait_ld(cur);
                for (int c0 = 0; c0 < nrows; c0 += 32) {
                    const bool more = c0 + 32 < nrows;
                    if (more) {
                        tmem_ld32_async(t0 + c0 + 32, nxt);
                    } else {
                        // every column of this accumulator is in registers: release it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (PAIR) mbar_arrive_cluster(tempty_leader + 8u * acc);
                            else mbar_arrive(&tempty_bar[acc]);
                        }
                    }
                    float a[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) a[c] = __uint_as_float(cur[c]);
                    if (W8 || A8) {
                        const float sa = A8 && c0 + lane < nrows ? scale_act[row0 + c0 + lane] : 1.0f;
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            a[c] *= sc;
                            if (A8) a[c] *= __shfl_sync(0xffffffffu, sa, c);
                        }
                    }
                    if (tma_store) {
                        // this warp's previous bulk store has finished reading the region
                        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                        __syncwarp();
                    }
                    if (tma_store && c0 + 32 <= nrows && fbase < Nout) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) box[c * 32 + lane] = a[c];
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        __syncwarp();
                        if (lane == 0) tma_store_2d(&tm_out, fbase, (int)((int64_t)ks * R + row0 + c0), box_s);
                    } else if (vec_ok) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) stage_t[lane][c] = a[c];
                        __syncwarp();
                        const int rr = lane >> 3, j = lane & 7;  // 4 rows x 8 feature quads per step
                        const int fv = fbase + 4 * j;
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int r = it * 4 + rr;
                            if (c0 + r < nrows && fv < Nout) {
                                const float4 v = make_float4(stage_t[4 * j + 0][r], stage_t[4 * j + 1][r],
                                                             stage_t[4 * j + 2][r], stage_t[4 * j + 3][r]);
                                *reinterpret_cast<float4 *>(outf + (size_t)(row0 + c0 + r) * ldo + fv) = v;
                            }
                        }
                        __syncwarp();
                    } else if (fbase + lane < Nout) {
                        float *dst = outf + (size_t)(row0 + c0) * ldo + fbase + lane;
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (c0 + c < nrows) dst[(size_t)c * ldo] = a[c];
                    }
                    if (more) {
                        tmem_wait_ld(nxt);
#pragma unroll
                        for (int c = 0; c < 32; ++c) cur[c] = nxt[c];
                    }
                }
            }
            if (SWIGLU) {  // (the plain epilogue released the accumulator after its last TMEM load)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR) mbar_arrive_cluster(tempty_leader + 8u * acc);  // the leader's barrier
                    else mbar_arrive(&tempty_bar[acc]);
                }
            }
            if (++acc == C::kAccBufs) { acc = 0; aphase ^= 1u; }
        }
        // bulk stores must have landed before the kernel's writes count as done
        if (!SWIGLU && tma_store && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        __syncwarp();
    }

    if (W8 && warp >= 6 && warp < 14) {
        // ------------------------------------------------------ converters (W8)
        // A warp may only reach its own quadrant of TMEM lanes (warp % 4), so converter warp
        // w takes rows [32 (w % 4), +32) -- one per lane -- and half kq = (w - 6) / 4 of
        // every 64-wide K block: per fp8 tile (two K blocks) it widens 2 x 32 values a lane
        // and stores them into the two K blocks' operand slots in TMEM.  The eight warps
        // run on their own (no barrier between them): each waits, converts and arrives.
        const int q = warp & 3, kq = (warp - 6) >> 2;
        const int crow = 32 * q + lane;
        const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(C::kASlot0 + 16 * kq);
        static_assert(!W8 || C::kStages > C::kABufs, "the activation ring must be deeper than the operand slots");
        int stage = 0, ab = 0;
        int64_t kbn = 0;  // K blocks of this CTA's sequence converted so far
        uint32_t phase = 0;
        bool stop = false;
        for (int item = unit; item < total && !stop; item += nunits) {
            int g, feat, ks, row0, row_end, kb0, kb1;
            decode(item, g, feat, ks, row0, row_end);
            kslice(ks, kb0, kb1);
            for (int kb = kb0; kb < kb1; kb += 2) {
                // one fp8 tile -> the operand slots of its two K blocks (ab, ab + 1).  Slot
                // reuse: K block n takes the slot of K block n - kABufs, free once that K
                // block's MMAs completed -- the commit on its activation stage's barrier
                // (the activation ring is deeper than kABufs, so that barrier cannot have
                // moved two phases past the one waited for)
                bool ok = mbar_wait(&ffull_bar[stage], phase, abort_flag);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t m = kbn + h - C::kABufs;  // the K block that last used the slot
                    if (m >= 0)
                        ok = ok && mbar_wait(&empty_bar[m % C::kStages], (uint32_t)((m / C::kStages) & 1), abort_flag);
                }
                if (!__all_sync(0xffffffffu, ok)) { stop = true; break; }
                tc_fence_after();
                uint32_t w0[16], w1[16];
                widen_e4m3_32(fring + stage * C::kW8Bytes, crow, 0, kq, w0);
                widen_e4m3_32(fring + stage * C::kW8Bytes, crow, 1, kq, w1);
                tmem_st16(tq + (uint32_t)(ab * C::kACols), w0);
                tmem_st16(tq + (uint32_t)((ab + 1) * C::kACols), w1);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&afull_bar[ab]);
                    mbar_arrive(&afull_bar[ab + 1]);
                    mbar_arrive(&fempty_bar[stage]);
                }
                ab += 2;
                kbn += 2;
                if (ab == C::kABufs) ab = 0;
                if (++stage == C::kFStages) { stage = 0; phase ^= 1u; }
            }
        }
        if (stop) { failed = true; *abort_flag = 1; }
    } else if (W8 && warp == 14 && lane == 0) {
        // ------------------------------------------------------ activation producer (W8)
        tma_prefetch_map(&tm_act);
        int stage = 0;
        uint32_t phase = 0;
        for (int item = unit; item < total && !failed; item += nunits) {
            int g, feat, ks, row0, row_end, kb0, kb1;
            decode(item, g, feat, ks, row0, row_end);
            kslice(ks, kb0, kb1);
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { failed = true; *abort_flag = 1; break; }
                mbar_arrive_expect_tx(&full_bar[stage], C::kBBytes);
                tma_2d<false>(stages + stage * C::kStageBytes, &tm_act, kb * kBK, row0, smem_u32(&full_bar[stage]));
                if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            }
        }
    }

    if (failed) set_device_error(dev_err, MOE_DEVERR_PIPELINE_TIMEOUT);
    __syncwarp();
    __syncthreads();
    if (PAIR) cluster_sync();  // no arrival from the peer can still be on its way
    if (*abort_flag) {
        // let copies and MMAs already in flight land before the CTA's memory is released
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) { }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_g<PAIR>(tmem_base, C::kTmemCols);
    }
}

// -------------------------------------------------------------------- host --
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// Weights [groups, Nout, K] bf16 as a 3-D map; box = 64 (K) x box_rows x 1 (group).
// Rows past Nout read as zero and never bleed into the next group.
bool encode_weight_map(CUtensorMap *m, const void *ptr, int groups, int Nout, int K, int box_rows)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)Nout, (cuuint64_t)groups};
    cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)Nout * (cuuint64_t)K * 2};
    cuuint32_t box[3] = {(cuuint32_t)kBK, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp8 (e4m3) weights [groups, Nout, K] as a 3-D byte map; box = 128 (K) x box_rows x 1:
// 128-byte rows (two 64-wide K blocks per load, the same bytes per row request as the
// bf16 tiles) with 128-byte swizzle.
bool encode_weight_map_fp8(CUtensorMap *m, const void *ptr, int groups, int Nout, int K, int box_rows)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)Nout, (cuuint64_t)groups};
    cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)Nout * (cuuint64_t)K};
    cuuint32_t box[3] = {(cuuint32_t)(2 * kBK), (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Activations [R, K] bf16 as a 2-D map; box = 64 (K) x box_rows; rows >= R read as zero.
bool encode_act_map(CUtensorMap *m, const void *ptr, int64_t R, int K, int box_rows)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)R};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// x [rows, K] bf16 as a 2-D map whose box is one row high (64 K values): the source of
// tile::gather4 loads of activation rows in any order.
bool encode_gather_map(CUtensorMap *m, const void *ptr, int64_t rows, int K)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, 1};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 output rows [rows, Nout] (row stride ldo elements) as a 2-D map for bulk stores:
// box = 32 features x 32 rows, no swizzle (the staging tile is a dense [32][32]).
bool encode_out_map_f32(CUtensorMap *m, void *ptr, int64_t rows, int Nout, int64_t ldo)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)Nout, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ldo * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Activations [R, K] e4m3 bytes as a 2-D byte map; box = 128 (K) x box_rows; rows >= R
// and K values past K read as zero.
bool encode_act_map_fp8(CUtensorMap *m, const void *ptr, int64_t R, int K, int box_rows)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)R};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)(2 * kBK), (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool SWIGLU, bool PAIR, bool W8, bool A8, bool GATHER = false>
cudaError_t launch_impl(const GroupedGemmArgs &a, cudaStream_t s)
{
    using C = Cfg<BN, SWIGLU, PAIR, W8, A8>;
    CUtensorMap ma, mb, mact;
    const int box_rows = SWIGLU ? kBM / 2 : kBM;
    auto enc_w = (W8 || A8) ? encode_weight_map_fp8 : encode_weight_map;
    if (!enc_w(&ma, a.w_a, a.groups, a.Nout, a.K, box_rows)) return cudaErrorInvalidValue;
    if (SWIGLU) {
        if (!enc_w(&mb, a.w_b, a.groups, a.Nout, a.K, box_rows)) return cudaErrorInvalidValue;
    } else {
        mb = ma;
    }
    if (GATHER) {
        if (!a.gather_rows || a.gather_src_rows < 1 || !encode_gather_map(&mact, a.act, a.gather_src_rows, a.K))
            return cudaErrorInvalidValue;
    } else {
        auto enc_act = A8 ? encode_act_map_fp8 : encode_act_map;
        if (!enc_act(&mact, a.act, a.R, a.K, C::kBRows)) return cudaErrorInvalidValue;
    }
    const int64_t ldo = a.ldo > 0 ? a.ldo : a.Nout;
    if (ldo < a.Nout) return cudaErrorInvalidValue;
    const int ks_out = SWIGLU ? 1 : (a.ksplit > 1 ? a.ksplit : 1);
    // plain GEMM: bulk tensor stores of the fp32 rows when the K slices' buffers sit one
    // after another (split_stride = R * ldo), the row stride is whole 16-byte units and
    // every row coordinate fits the map's 32-bit coordinates
    CUtensorMap mout = ma;
    int tma_store = 0;
    if (!SWIGLU && a.out && (ldo & 3) == 0 && (a.Nout & 31) == 0 &&
        (ks_out == 1 || a.split_stride == a.R * ldo) && (int64_t)ks_out * a.R < (int64_t(1) << 31) &&
        (reinterpret_cast<uintptr_t>(a.out) & 15) == 0)
        tma_store = encode_out_map_f32(&mout, a.out, (int64_t)ks_out * a.R, a.Nout, ldo) ? 1 : 0;
    auto kern = grouped_gemm_kernel<BN, SWIGLU, PAIR, W8, A8, GATHER>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (err != cudaSuccess) return err;
    const int ksplit = SWIGLU ? 1 : (a.ksplit > 1 ? a.ksplit : 1);
    const int sms = device_sm_count();
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    cfg.gridDim = dim3((unsigned)(PAIR ? (sms / 2) * 2 : sms));
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = PAIR ? 2 : 1;
    err = cudaLaunchKernelEx(&cfg, kern, ma, mb, mact, a.offsets, a.groups, a.rows_single, a.R, a.K, a.Nout, a.out,
                             ksplit, a.split_stride, a.scale_a, a.scale_b, a.scale_act, ldo, a.gather_rows, mout,
                             tma_store, a.ends, a.dev_err);
    if (err != cudaSuccess) return err;
    count_launch();
    return cudaGetLastError();
}

// Expected work items on CTA pairs, from the mean group size (the true count is only
// known on the device).
int64_t gemm_pair_tiles(int64_t R, int groups, int Nout, bool swiglu, int ksplit)
{
    const int bn = gemm_choose_token_tile(R, groups, swiglu);
    const int64_t active = R < groups ? R : groups;
    if (active <= 0) return 0;
    const int64_t mean = (R + active - 1) / active;
    const int feat = swiglu ? kBM : 2 * kBM;  // output features per pair tile
    return active * ((mean + bn - 1) / bn) * ((Nout + feat - 1) / feat) * (ksplit > 1 ? ksplit : 1);
}

template <bool SWIGLU, bool W8, bool A8>
cudaError_t launch_dispatch(const GroupedGemmArgs &a, cudaStream_t s)
{
    if (a.groups < 1 || a.groups > kMaxGroups) return cudaErrorInvalidValue;
    if (SWIGLU && (a.Nout % (kBM / 2)) != 0) return cudaErrorInvalidValue;  // whole 64-feature tiles
    const int bn = a.token_tile ? a.token_tile : gemm_choose_token_tile(a.R, a.groups, SWIGLU);
    // Tiles run on CTA pairs (M = 256 weight rows per MMA): each SM streams half the
    // token tile, and the pair reads each activation tile once per 256 weight rows
    // instead of once per 128.  A tiny batch whose pair tiles would not even cover the
    // SM pairs once runs single-CTA tiles instead (twice the tiles, every SM streaming).
    if (W8 && !A8) {
        // fp8 weights widened on chip: single-CTA tiles.  A pair's MMA would read converted operands from
        // the other CTA, which then has to signal every K step across the cluster.
        // (token tiles up to 128 rows: two 256-column accumulators and the operand slots
        // would not fit in TMEM's 512 columns)
        switch (bn) {
            case 32: return launch_impl<32, SWIGLU, false, true, false>(a, s);
            case 64: return launch_impl<64, SWIGLU, false, true, false>(a, s);
            case 96:
            case 128:
            case 192:
            case 256: return launch_impl<128, SWIGLU, false, true, false>(a, s);
            default: return cudaErrorInvalidValue;
        }
    } else {
        if constexpr (!SWIGLU && !W8 && !A8) {
            // single-CTA tiles on request: an operand of at most 128 rows (a pair's M = 256
            // would multiply rows of zeros)
            if (a.single_cta) {
                switch (bn) {
                    case 32: return launch_impl<32, false, false, false, false>(a, s);
                    case 64: return launch_impl<64, false, false, false, false>(a, s);
                    case 128: return launch_impl<128, false, false, false, false>(a, s);
                    default: return cudaErrorInvalidValue;
                }
            }
        }
        if constexpr (SWIGLU && !A8) {
            // activation rows gathered from x through the row map (no permuted copy)
            if (a.gather_rows) {
                if (bn <= 64 && gemm_pair_tiles(a.R, a.groups, a.Nout, SWIGLU, a.ksplit) < device_sm_count() / 2) {
                    switch (bn) {
                        case 32: return launch_impl<32, true, false, false, false, true>(a, s);
                        case 64: return launch_impl<64, true, false, false, false, true>(a, s);
                    }
                }
                switch (bn) {
                    case 32: return launch_impl<32, true, true, false, false, true>(a, s);
                    case 64: return launch_impl<64, true, true, false, false, true>(a, s);
                    case 96: return launch_impl<96, true, true, false, false, true>(a, s);
                    case 128: return launch_impl<128, true, true, false, false, true>(a, s);
                    case 192: return launch_impl<192, true, true, false, false, true>(a, s);
                    case 256: return launch_impl<256, true, true, false, false, true>(a, s);
                    default: return cudaErrorInvalidValue;
                }
            }
        }
        if (a.gather_rows) return cudaErrorInvalidValue;  // gathering is a bf16 SwiGLU option only
        if (bn <= 64 && gemm_pair_tiles(a.R, a.groups, a.Nout, SWIGLU, a.ksplit) < device_sm_count() / 2) {
            switch (bn) {
                case 32: return launch_impl<32, SWIGLU, false, false, A8>(a, s);
                case 64: return launch_impl<64, SWIGLU, false, false, A8>(a, s);
            }
        }
        switch (bn) {
            case 32: return launch_impl<32, SWIGLU, true, false, A8>(a, s);
            case 64: return launch_impl<64, SWIGLU, true, false, A8>(a, s);
            case 96: return launch_impl<96, SWIGLU, true, false, A8>(a, s);
            case 128: return launch_impl<128, SWIGLU, true, false, A8>(a, s);
            case 192: return launch_impl<192, SWIGLU, true, false, A8>(a, s);
            case 256: return launch_impl<256, SWIGLU, true, false, A8>(a, s);
            default: return cudaErrorInvalidValue;
        }
    }
}

}  // namespace

int device_sm_count()
{
    static int counts[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && counts[dev] > 0) return counts[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) counts[dev] = n;
    return n;
}

// Token tile from the expected largest group.  The MMA width follows each tile's rows,
// so a wide tile wastes no tensor work on a short group; what a wide tile costs is
// shared memory (fewer pipeline stages, so fewer weight bytes in flight from HBM).
// Groups should fit in one tile where possible, so each weight tile streams through
// shared memory once: the tile covers the mean rows per group plus three standard
// deviations of a balanced routing (mean + 3 sqrt(mean)), rounded up to the tiles
// compiled (32, 64, 96, 128, 192, 256).
int gemm_choose_token_tile(int64_t R, int groups, bool swiglu)
{
    (void)swiglu;
    const double mean = (double)R / (groups > 0 ? groups : 1);
    const double want = mean + 3.0 * std::sqrt(mean);
    static const int tiles[] = {32, 64, 96, 128, 192, 256};
    for (int t : tiles)
        if (want <= t) return t;
    return 256;
}

// K slices for the W2 GEMM of a decode-shaped layer: when the tiles (estimated from
// the mean group size) cover the SMs in few waves with a ragged last one, split K so
// the last wave is nearly full.  1 for everything with enough tiles.
int gemm2_ksplit(int64_t R, int groups, int K, int Nout)
{
    const int units = device_sm_count() / 2;  // CTA pairs
    const int bn = gemm_choose_token_tile(R, groups, false);
    if (bn >= 128) return 1;  // large groups: enough work per tile
    const int64_t tiles = gemm_pair_tiles(R, groups, Nout, false, 1);
    if (tiles <= 0 || tiles >= 4 * (int64_t)units) return 1;
    int best = 1;
    double best_eff = 0.0;
    for (int ks = 1; ks <= 4; ++ks) {
        if (K / kBK < 6 * ks) break;  // keep every slice at least 6 K-blocks long
        const int64_t n = tiles * ks;
        const double eff = (double)n / (double)(((n + units - 1) / units) * units);
        if (eff > best_eff + 0.02) { best_eff = eff; best = ks; }
    }
    return best;
}

cudaError_t launch_gemm13_swiglu(const GroupedGemmArgs &a, cudaStream_t s)
{
    if (a.w8 && (!a.scale_a || !a.scale_b)) return cudaErrorInvalidValue;
    if (a.a8 && (!a.w8 || !a.scale_act)) return cudaErrorInvalidValue;
    if (a.a8) return launch_dispatch<true, false, true>(a, s);
    return a.w8 ? launch_dispatch<true, true, false>(a, s) : launch_dispatch<true, false, false>(a, s);
}

cudaError_t launch_gemm2(const GroupedGemmArgs &a, cudaStream_t s)
{
    if (a.w8 && !a.scale_a) return cudaErrorInvalidValue;
    if (a.a8 && (!a.w8 || !a.scale_act)) return cudaErrorInvalidValue;
    if (a.a8) return launch_dispatch<false, false, true>(a, s);
    return a.w8 ? launch_dispatch<false, true, false>(a, s) : launch_dispatch<false, false, false>(a, s);
}

}  // namespace moe
