// grouped_mx.cu -- the expert FFN of the MXFP8 variant on sm_100a tensor
// cores: E4M3 operands with one UE8M0 (power-of-two) scale per 32 values
// along K, applied by the tensor core itself (tcgen05.mma kind::mxf8f6f4
// block_scale).  The pages name an MXFP8 MoE runtime only as not yet
// qualified ("Exact AVX2 FP8 arithmetic conversion avoids costly LUT
// gathers", "Real-checkpoint measurements", caveats); the arithmetic follows
// the OCP Microscaling Formats (the repository's MX readings).
//
// Unlike the 128x128-block path, no K block needs its own accumulator: the
// scales are inside the MMA, so each tile accumulates over all of K in one
// TMEM buffer and is drained once.
//
// Launch sequence of one moe_grouped_ffn_mx call (stream-ordered):
//   gather   : A code rows and their scale bytes in expert order
//   gate/up  : tile 128 rows x (96 gate + 96 up) columns; epilogue
//              h = SiLU(g) * u, MX-requantised per 32 columns
//   down     : tile 128 rows x 192 output columns; epilogue y[pair] = w * o
// N = 192 is the widest tile for which two accumulators and the scale ring
// fit the 512 TMEM columns; it reads 40 KB of operands per 128-deep K block
// for 6.3 MFLOP, so the tensor pipe, not the shared-memory fill, sets the
// pace of a K block.
//
// Warp roles (384 threads, one CTA per SM, persistent over work items ordered
// expert-major, then n-tile, then m-tile):
//   warp 0      weight TMA producers (lanes 0, 1: one 96-row half each)
//   warp 1      MMA issuer (one lane; also allocates TMEM)
//   warp 3      activation TMA producers (lanes 0, 1: one 64-row half each)
//   warps 4..7  epilogue: warp w drains TMEM lanes 32*(w%4), once per item
//   warp 2      scale loader (all lanes): the tile's A and B scale bytes of
//               each K block from global memory into a shared ring, four K
//               blocks per 16-byte load, the next group's loads in flight
//   warps 8..11 scale writers: per K block, copy the shared slot into a
//               TMEM ring with tcgen05.st.  The MMA reads a row's scale from
//               the lane of that row in every 32-lane sub-partition, so each
//               of the four warps writes the same data into its own
//               sub-partition.  A tcgen05 wait also waits for the warp's
//               outstanding global loads, hence the split: the writers keep
//               none in flight.
// TMEM: two 192-column accumulators (items alternate) and SF_SLOTS slots of
// 16 scale columns.  Scale layout (K block of 128 = 4 chunks of 32): row m of
// the A tile -> lanes m%32 (+32 per sub-partition), slot column m/32, byte
// j = chunk j; B row n likewise in the slot's columns 8 + n/32.  The MMA of
// chunk j selects byte j (scale-factor id j).
// Every wait is bounded (2 s); on expiry the CTA raises an abort flag, records
// MOE_DEV_WAIT_TIMEOUT and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>

#include "internal.h"
#include "mx_rule.cuh"
#include "sm100.cuh"

namespace fp8moe {
namespace {

using namespace sm100;

constexpr int MX_BM = 128;
constexpr int MX_BN = 192;            // MMA N: output columns of a tile
constexpr int MX_HALF = MX_BN / 2;    // gate/up: 96 gate + 96 up weight rows
constexpr int MX_BK = 128;
constexpr int MX_STAGES = 5;
constexpr int MX_A_TILE = MX_BM * MX_BK;  // 16 KiB
constexpr int MX_B_TILE = MX_BN * MX_BK;  // 24 KiB
constexpr int MX_STAGE = MX_A_TILE + MX_B_TILE;
constexpr int MX_THREADS = 384;
constexpr int SF_SLOTS = 8;
constexpr int SF_SLOT_COLS = 16;              // A: columns 0..3, B: columns 8..13
constexpr int SF_COL = 2 * MX_BN;             // the scale ring follows the two accumulators
constexpr uint32_t MX_TMEM_COLS = 512;
constexpr uint64_t MX_WAIT_NS = 2000000000ull;
constexpr int MX_MAX_E = 1024;

constexpr int MB_FULL = 0;                       // [stages]: both producers (arrive + tx)
constexpr int MB_EMPTY = MB_FULL + MX_STAGES;    // [stages]: MMA commit
constexpr int MB_SFF = MB_EMPTY + MX_STAGES;     // [slots]: the four stager warps
constexpr int MB_SFE = MB_SFF + SF_SLOTS;        // [slots]: MMA commit
constexpr int SG_SLOTS = 3;                      // shared ring of scale groups (four K blocks each)
constexpr int MB_SSF = MB_SFE + SF_SLOTS;        // [SG_SLOTS]: the loader's 32 lanes' copies landed
constexpr int MB_SSE = MB_SSF + SG_SLOTS;        // [SG_SLOTS]: the four writers read the group
constexpr int MB_AF = MB_SSE + SG_SLOTS;         // [2]: accumulator full (MMA commit)
constexpr int MB_AE = MB_AF + 2;                 // [2]: accumulator drained (four epilogue warps)
constexpr int MB_N = MB_AE + 2;
constexpr int SF_WORDS = 10;                   // per lane and K block: 4 A + 6 B scale words
constexpr int SG_BYTES = SF_WORDS * 32 * 16;   // one group: [word][lane][4 K blocks] 32-bit words
constexpr int MX_OFF_SFS = MX_STAGES * MX_STAGE;  // shared ring of scale groups
constexpr int MX_OFF_BARS = MX_OFF_SFS + SG_SLOTS * SG_BYTES;
constexpr int MX_OFF_MISC = MX_OFF_BARS + MB_N * 8;
constexpr int MX_OFF_SEG = MX_OFF_MISC + 16;  // [E+1] offsets, then [E+1] item prefix
constexpr int mx_smem_bytes(int E) { return MX_OFF_SEG + 2 * (E + 1) * 4 + 1024; }
static_assert(SF_COL + SF_SLOTS * SF_SLOT_COLS <= static_cast<int>(MX_TMEM_COLS), "scale ring exceeds TMEM");
static_assert(MX_STAGE % 1024 == 0 && MX_A_TILE % 1024 == 0 && (MX_HALF * 128) % 1024 == 0,
              "128-byte-swizzled tiles need 1024-byte alignment");

struct MxParams {
    int E;
    int num_kb;            // K blocks of 128
    int num_groups;        // groups of four K blocks: ceil(num_kb / 4)
    int n_tiles;           // output tiles per expert
    int64_t P;             // rows of the pair buffers (T * top_k)
    const int32_t* offsets;
    const uint8_t* a_sf;   // A rows' scale bytes (expert order), K-group-major:
                           // [ceil(K/512)][P][16], 16 = four K blocks of four chunks
    int a_chunks;          // valid 32-column chunks of an A row (K / 32)
    const uint8_t* b_sf0;  // gate/up: s_gate; down: s_down, packed [E][ceil(K/512)][b_rows][16]
    const uint8_t* b_sf1;  // gate/up: s_up
    int b_rows;            // weight rows per expert (I or H)
    int b_chunks;          // valid chunks of a weight row (K / 32)
    // gate/up epilogue
    uint8_t* h_codes;      // [P, Ip]
    uint8_t* h_scales;     // [ceil(Ip/512)][P][16], the layout of a_sf
    int Ip;
    int I;
    // down epilogue
    const int32_t* sorted_pairs;
    const float* topk_w;
    float* y;              // [P, H]
    int H;
    int* status;
};

struct MxItem {
    int e, nt, mt;
};

__device__ __forceinline__ MxItem mx_decode(const int* seg, const int* ipre, int E, int item)
{
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ipre[mid] <= item) lo = mid;
        else hi = mid;
    }
    MxItem it;
    it.e = lo;
    const int local = item - ipre[lo];
    const int mts = (seg[lo + 1] - seg[lo] + MX_BM - 1) / MX_BM;
    it.nt = local / mts;
    it.mt = local - it.nt * mts;
    return it;
}

// Instruction descriptor, kind::mxf8f6f4 with block scaling: A and B E4M3,
// both K-major, D FP32, UE8M0 scales, shape M x N; scale-factor ids select
// the byte of the scale columns (the K chunk).
__device__ __forceinline__ uint32_t idesc_mx(int M, int N, uint32_t sf_id)
{
    return (sf_id << 4)                               // B scale-factor id
           | (0u << 7) | (0u << 10)                   // A, B format E4M3
           | (0u << 15) | (0u << 16)                  // A, B K-major
           | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
           | (1u << 23)                               // scale format UE8M0
           | (static_cast<uint32_t>(M >> 4) << 24)    // M / 16
           | (sf_id << 29);                           // A scale-factor id
}

// D[tmem] (+)= A[smem] * B[smem]^T with the block scales in TMEM.
__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_st32x8(uint32_t taddr, const uint32_t (&v)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- roles

// Weight producers (warp 0, lanes 0 and 1) and activation producers (warp 3,
// lanes 0 and 1): each lane loads one half of its operand's tile per K
// block (gate or up rows, the first or second 96 down rows; the first or
// second 64 activation rows), and a stage is full when all four halves have
// landed.  The TMA unit serves each issuing thread's requests one after
// another, about 25 bytes per clock per thread (measured), so one thread
// per 24 KB weight tile would pace the K loop.
template <int MODE>
__device__ __forceinline__ void mx_producer_b(const CUtensorMap* tm0, const CUtensorMap* tm1, const MxParams& p,
                                              const int* seg, const int* ipre, int total, uint32_t sbase,
                                              uint32_t bars, volatile int* abort, int part)
{
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
        const MxItem w = mx_decode(seg, ipre, p.E, item);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const int s = it % MX_STAGES;
            if (!mbar_wait_bounded(bars + 8 * (MB_EMPTY + s), ((it / MX_STAGES) & 1) ^ 1, abort, MX_WAIT_NS)) {
                ok = false;
                break;
            }
            const uint32_t fb = bars + 8 * (MB_FULL + s);
            mbar_arrive_expect_tx(fb, MX_B_TILE / 2);
            const uint32_t dst = sbase + s * MX_STAGE + MX_A_TILE + part * (MX_B_TILE / 2);
            if (MODE == 0)  // 96 gate rows, then 96 up rows, of n-tile nt
                tma_load_3d(dst, part ? tm1 : tm0, kb * MX_BK, w.nt * MX_HALF, w.e, fb);
            else
                tma_load_3d(dst, tm0, kb * MX_BK, w.nt * MX_BN + part * MX_HALF, w.e, fb);
        }
    }
    if (!ok) {  // let the copies already issued land before the CTA can exit
        for (int j = it - MX_STAGES > 0 ? it - MX_STAGES : 0; j < it; ++j) {
            volatile int no_abort = 0;
            mbar_wait_bounded(bars + 8 * (MB_FULL + j % MX_STAGES), (j / MX_STAGES) & 1, &no_abort, MX_WAIT_NS / 4);
        }
    }
}

__device__ __forceinline__ void mx_producer_a(const CUtensorMap* tmA, const MxParams& p, const int* seg,
                                              const int* ipre, int total, uint32_t sbase, uint32_t bars,
                                              volatile int* abort, int part)
{
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
        const MxItem w = mx_decode(seg, ipre, p.E, item);
        const int row0 = seg[w.e] + w.mt * MX_BM;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const int s = it % MX_STAGES;
            if (!mbar_wait_bounded(bars + 8 * (MB_EMPTY + s), ((it / MX_STAGES) & 1) ^ 1, abort, MX_WAIT_NS)) {
                ok = false;
                break;
            }
            const uint32_t fb = bars + 8 * (MB_FULL + s);
            mbar_arrive_expect_tx(fb, MX_A_TILE / 2);
            tma_load_2d(sbase + s * MX_STAGE + part * (MX_A_TILE / 2), tmA, kb * MX_BK, row0 + part * (MX_BM / 2), fb);
        }
    }
    if (!ok) {
        for (int j = it - MX_STAGES > 0 ? it - MX_STAGES : 0; j < it; ++j) {
            volatile int no_abort = 0;
            mbar_wait_bounded(bars + 8 * (MB_FULL + j % MX_STAGES), (j / MX_STAGES) & 1, &no_abort, MX_WAIT_NS / 4);
        }
    }
}

// Scale words for lane t: the A scales of tile rows t, t+32, t+64, t+96
// (words 0..3) and the B scales of rows t, t+32, .., t+160 (words 4..9),
// four K chunks (one K block) per 32-bit word.  Both operands' scales are
// K-group-major ([groups][rows][16 bytes], a group = four K blocks), so the
// loader fetches a group of four K blocks of 32 consecutive rows with one
// coalesced 16-byte-per-lane copy.  A cursor walks this CTA's (item, group)
// sequence.
struct SfGroup {
    int item, kb0, row0;
    MxItem w;
};

__device__ __forceinline__ void sf_group_next(SfGroup& c, const MxParams& p, const int* seg, const int* ipre,
                                              int total)
{
    c.kb0 += 4;
    if (c.kb0 < p.num_kb) return;
    c.kb0 = 0;
    c.item += gridDim.x;
    if (c.item < total) {
        c.w = mx_decode(seg, ipre, p.E, c.item);
        c.row0 = seg[c.w.e] + c.w.mt * MX_BM;
    }
}

// Chunks at or beyond nvalid of the 32-bit word of K block kb (chunks 4kb ..
// 4kb+3) read as 127 (2^0): K padding, whose codes are zero.
__device__ __forceinline__ uint32_t mask_sf4(uint32_t w, int kb, int nvalid)
{
    const int c0 = 4 * kb;
    if (c0 + 4 <= nvalid) return w;
#pragma unroll
    for (int b = 0; b < 4; ++b)
        if (c0 + b >= nvalid) w = (w & ~(0xFFu << (8 * b))) | (0x7Fu << (8 * b));
    return w;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Scale loader (warp 2, all lanes): per group of four K blocks, lane t
// copies the 16-byte group words of A rows t + 32j (j < 4) and B rows
// t + 32j (j < 6) straight into shared slot g % SG_SLOTS with cp.async, laid
// out [word][lane][16 B], and the copies' completion arrives on the slot's
// barrier (no registers in between, so three groups are in flight).  Rows
// past the weights are zero-filled (a finite scale for zero codes).  The
// loader issues no tcgen05 operation: a tcgen05 wait also waits for the
// warp's outstanding global loads, so the warps that write TMEM keep none.
template <int MODE>
__device__ __forceinline__ void mx_sf_loader(const MxParams& p, const int* seg, const int* ipre, int total,
                                             uint32_t sfs, uint32_t bars, volatile int* abort)
{
    const int lane = threadIdx.x & 31;
    if (static_cast<int>(blockIdx.x) >= total) return;
    SfGroup c;
    c.item = blockIdx.x;
    c.kb0 = 0;
    c.w = mx_decode(seg, ipre, p.E, c.item);
    c.row0 = seg[c.w.e] + c.w.mt * MX_BM;
    for (int g = 0; c.item < total; ++g) {
        const int slot = g % SG_SLOTS;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars + 8 * (MB_SSE + slot), ((g / SG_SLOTS) & 1) ^ 1, abort,
                                                        MX_WAIT_NS)))
            break;
        const uint32_t dst = sfs + slot * SG_BYTES + lane * 16;
        const int grp = c.kb0 >> 2;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int64_t m = c.row0 + lane + 32 * j;
            m = m < p.P ? m : p.P - 1;
            cp_async16(dst + j * 512, p.a_sf + (static_cast<int64_t>(grp) * p.P + m) * 16, 16);
        }
#pragma unroll
        for (int j = 0; j < 6; ++j) {
            const uint8_t* base;
            int row;
            if (MODE == 0) {  // B rows 0..95 gate, 96..191 up
                base = j < 3 ? p.b_sf0 : p.b_sf1;
                row = c.w.nt * MX_HALF + lane + 32 * (j % 3);
            } else {
                base = p.b_sf0;
                row = c.w.nt * MX_BN + lane + 32 * j;
            }
            const bool in = row < p.b_rows;
            const int64_t gw = (static_cast<int64_t>(c.w.e) * p.num_groups + grp) * p.b_rows + (in ? row : 0);
            cp_async16(dst + (4 + j) * 512, base + gw * 16, in ? 16u : 0u);
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bars + 8 * (MB_SSF + slot))
                     : "memory");
        sf_group_next(c, p, seg, ipre, total);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Scale writers (warps 8..11, all lanes): per group, read this lane's words
// of its four K blocks from the shared slot and release the slot; then per
// K block, once the MMAs that read the TMEM slot's previous contents are
// done, write TMEM lane 32q + t of TMEM slot it % SF_SLOTS (columns 0..3 A
// rows t + 32j, columns 8..13 B rows t + 32j) and hand it to the issuer.
__device__ __forceinline__ void mx_sf_writer(const MxParams& p, int n_items, uint32_t sfs, uint32_t bars,
                                             uint32_t tmem, volatile int* abort)
{
    const int lane = threadIdx.x & 31;
    const int q = (threadIdx.x >> 5) & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int it = 0, g = 0;
    for (int item = 0; item < n_items; ++item) {
        for (int kb0 = 0; kb0 < p.num_kb; kb0 += 4, ++g) {
            const int slot = g % SG_SLOTS;
            if (!__all_sync(0xFFFFFFFFu,
                            mbar_wait_bounded(bars + 8 * (MB_SSF + slot), (g / SG_SLOTS) & 1, abort, MX_WAIT_NS)))
                return;
            const int nk = p.num_kb - kb0 < 4 ? p.num_kb - kb0 : 4;
            uint32_t v[SF_WORDS][4];
            const uint32_t src = sfs + slot * SG_BYTES + lane * 16;
#pragma unroll
            for (int j = 0; j < SF_WORDS; ++j)
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v[j][0]), "=r"(v[j][1]), "=r"(v[j][2]), "=r"(v[j][3])
                             : "r"(src + j * 512)
                             : "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + 8 * (MB_SSE + slot));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i >= nk) break;
                const int kb = kb0 + i;
                const int ss = it % SF_SLOTS;
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars + 8 * (MB_SFE + ss), ((it / SF_SLOTS) & 1) ^ 1,
                                                                abort, MX_WAIT_NS)))
                    return;
                tc_fence_after();
                uint32_t a[8], b[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) a[j] = mask_sf4(v[j][i], kb, p.a_chunks);
                a[4] = a[5] = a[6] = a[7] = 0u;
#pragma unroll
                for (int j = 0; j < 6; ++j) b[j] = mask_sf4(v[4 + j][i], kb, p.b_chunks);
                b[6] = b[7] = 0u;
                const uint32_t col = lane_base + SF_COL + ss * SF_SLOT_COLS;
                tmem_st32x8(col, a);
                tmem_st32x8(col + 8, b);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + 8 * (MB_SFF + ss));
                ++it;
            }
        }
    }
}

// MMA issuer (one lane): per item, wait until the accumulator buffer of the
// item's parity is drained; per K block, wait for the operand stage and the
// scale slot, issue four N = 192, K = 32 block-scaled MMAs (chunk j reads
// byte j of the scale columns), and commit so that the stage and the slot are
// released when those MMAs are done; after the item's last K block, commit
// the accumulator to the epilogue.
__device__ __forceinline__ void mx_mma(const MxParams& p, const int* seg, const int* ipre, int total, uint32_t sbase,
                                       uint32_t bars, uint32_t tmem, volatile int* abort)
{
    int it = 0, nitem = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x, ++nitem) {
        const int b = nitem & 1;
        if (!mbar_spin_bounded(bars + 8 * (MB_AE + b), ((nitem >> 1) & 1) ^ 1, abort, MX_WAIT_NS)) goto drain;
        tc_fence_after();
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const int s = it % MX_STAGES, ss = it % SF_SLOTS;
            if (!mbar_spin_bounded(bars + 8 * (MB_FULL + s), (it / MX_STAGES) & 1, abort, MX_WAIT_NS) ||
                !mbar_spin_bounded(bars + 8 * (MB_SFF + ss), (it / SF_SLOTS) & 1, abort, MX_WAIT_NS))
                goto drain;
            tc_fence_after();
            {
                const uint32_t a_addr = sbase + s * MX_STAGE;
                const uint32_t b_addr = a_addr + MX_A_TILE;
                const uint32_t d = tmem + b * MX_BN;
                const uint32_t sfa = tmem + SF_COL + ss * SF_SLOT_COLS;
                const uint32_t sfb = sfa + 8;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_mx(d, sw128_kmajor_desc(a_addr + j * 32), sw128_kmajor_desc(b_addr + j * 32),
                           idesc_mx(MX_BM, MX_BN, static_cast<uint32_t>(j)), sfa | (static_cast<uint32_t>(j) << 30),
                           sfb | (static_cast<uint32_t>(j) << 30), (kb > 0 || j > 0) ? 1u : 0u);
                mma_commit(bars + 8 * (MB_EMPTY + s));
                mma_commit(bars + 8 * (MB_SFE + ss));
            }
        }
        mma_commit(bars + 8 * (MB_AF + b));
    }
    return;
drain:
    // wait for the MMAs already issued before TMEM is released: the last
    // slot commit tracks every MMA this thread issued
    if (it > 0) {
        volatile int no_abort = 0;
        const int j = it - 1;
        mbar_wait_bounded(bars + 8 * (MB_SFE + j % SF_SLOTS), (j / SF_SLOTS) & 1, &no_abort, MX_WAIT_NS / 4);
    }
}

// SiLU(g) * u with the hardware exp2 and reciprocal approximations, the
// formula of the 128x128-block path's epilogue.
__device__ __forceinline__ float silu_mul(float g, float u)
{
    const float e = ex2_approx_ftz(-g * 1.4426950408889634f);
    return (g * rcp_approx_ftz(1.0f + e)) * u;
}

// Epilogue (warps 4..7): thread = one row of the tile (TMEM lane 32q + lane).
//   gate/up: columns [0,96) hold g, [96,192) u of intermediate columns
//            nt*96 .. nt*96+95; h = SiLU(g) * u; each 32 columns are one
//            MX block of the intermediate row: scale byte and 32 codes.
//   down:    y[pair, nt*192 + c] = topk_w[pair] * acc[c] for c < 192.
// The accumulator is released after its last TMEM load, before the last
// block's arithmetic and stores.
template <int MODE>
__device__ __forceinline__ void mx_epilogue(const MxParams& p, const int* seg, const int* ipre, int total,
                                            uint32_t bars, uint32_t tmem, volatile int* abort)
{
    const int lane = threadIdx.x & 31;
    const int q = (threadIdx.x >> 5) & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int nitem = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x, ++nitem) {
        const MxItem w = mx_decode(seg, ipre, p.E, item);
        const int b = nitem & 1;
        const int r = seg[w.e] + w.mt * MX_BM + q * 32 + lane;
        const bool valid = r < seg[w.e + 1];
        int pair = -1;
        if (MODE == 1 && valid) pair = __ldg(p.sorted_pairs + r);  // in flight during the wait
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars + 8 * (MB_AF + b), (nitem >> 1) & 1, abort, MX_WAIT_NS)))
            return;
        tc_fence_after();
        const uint32_t col = lane_base + b * MX_BN;
        if (MODE == 0) {
#pragma unroll 1
            for (int blk = 0; blk < MX_HALF / 32; ++blk) {
                uint32_t g[32], u[32];
                __syncwarp();  // the loads are warp-collective
                tmem_ld32_issue(col + blk * 32, g);
                tmem_ld_wait(g);
                tmem_ld32_issue(col + MX_HALF + blk * 32, u);
                tmem_ld_wait(u);
                if (blk == MX_HALF / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars + 8 * (MB_AE + b));
                }
                const int c0 = w.nt * MX_HALF + blk * 32;  // intermediate column of this block
                if (!valid || c0 >= p.I) continue;
                float h[32];
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    h[i] = silu_mul(__uint_as_float(g[i]), __uint_as_float(u[i]));
                    amax = fmax_nan(amax, fabsf(h[i]));
                }
                uint8_t* dst = p.h_codes + static_cast<int64_t>(r) * p.Ip + c0;
                uint8_t sc;
                uint4 o0, o1;
                if (!isfinite(amax)) {
                    sc = 0xFF;
                    o0 = o1 = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
                } else {
                    const int se = mx::shared_exponent(amax);
                    sc = static_cast<uint8_t>(se + 127);
                    const float f = mx::inv_scale(se);
                    uint32_t wv[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        wv[j] = e4m3x2(h[4 * j] * f, h[4 * j + 1] * f) | (e4m3x2(h[4 * j + 2] * f, h[4 * j + 3] * f) << 16);
                    o0 = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    o1 = make_uint4(wv[4], wv[5], wv[6], wv[7]);
                }
                reinterpret_cast<uint4*>(dst)[0] = o0;
                reinterpret_cast<uint4*>(dst)[1] = o1;
                p.h_scales[((static_cast<int64_t>(c0) >> 9) * p.P + r) * 16 + ((c0 >> 5) & 15)] = sc;
            }
        } else {
            float wt = 0.f;
            if (pair >= p.P || (valid && pair < 0)) {
                atomicOr(p.status, kDevBadPair);
                pair = -1;
            } else if (pair >= 0) {
                wt = __ldg(p.topk_w + pair);
            }
            float* dst = pair >= 0 ? p.y + static_cast<int64_t>(pair) * p.H + w.nt * MX_BN : nullptr;
#pragma unroll 1
            for (int c = 0; c < MX_BN / 32; ++c) {
                uint32_t v[32];
                __syncwarp();
                tmem_ld32_issue(col + c * 32, v);
                tmem_ld_wait(v);
                if (c == MX_BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars + 8 * (MB_AE + b));
                }
                if (!dst || w.nt * MX_BN + c * 32 >= p.H) continue;
                float4* g4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    g4[i] = make_float4(wt * __uint_as_float(v[4 * i]), wt * __uint_as_float(v[4 * i + 1]),
                                        wt * __uint_as_float(v[4 * i + 2]), wt * __uint_as_float(v[4 * i + 3]));
            }
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(MX_THREADS, 1)
    grouped_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                      const __grid_constant__ CUtensorMap tmB1, const MxParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + MX_OFF_BARS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MX_OFF_MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + MX_OFF_MISC + 4);
    int* bad = reinterpret_cast<int*>(smem + MX_OFF_MISC + 8);
    int* seg = reinterpret_cast<int*>(smem + MX_OFF_SEG);
    int* ipre = seg + (p.E + 1);
    const int warp = threadIdx.x >> 5;
    const int E = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < MX_STAGES; ++s) {
            mbar_init(bars + 8 * (MB_FULL + s), 4);   // four producer lanes: arrive + tx
            mbar_init(bars + 8 * (MB_EMPTY + s), 1);  // MMA commit
        }
        for (int s = 0; s < SF_SLOTS; ++s) {
            mbar_init(bars + 8 * (MB_SFF + s), 4);    // four writer warps
            mbar_init(bars + 8 * (MB_SFE + s), 1);    // MMA commit
        }
        for (int s = 0; s < SG_SLOTS; ++s) {
            mbar_init(bars + 8 * (MB_SSF + s), 32);   // the loader's 32 lanes (cp.async completion)
            mbar_init(bars + 8 * (MB_SSE + s), 4);    // four writer warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars + 8 * (MB_AF + b), 1);     // MMA commit
            mbar_init(bars + 8 * (MB_AE + b), 4);     // four epilogue warps
        }
        *abort = 0;
        *bad = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB0);
        prefetch_tmap(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), MX_TMEM_COLS);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i <= E; i += blockDim.x) seg[i] = __ldg(p.offsets + i);
    __syncthreads();
    if (threadIdx.x == 0) {
        int okv = (seg[0] == 0);
        int acc = 0;
        ipre[0] = 0;
        for (int e = 0; e < E; ++e) {
            const int c = seg[e + 1] - seg[e];
            if (c < 0 || seg[e + 1] > p.P) okv = 0;
            acc += (c > 0 ? (c + MX_BM - 1) / MX_BM : 0) * p.n_tiles;
            ipre[e + 1] = acc;
        }
        if (!okv) {
            *bad = 1;
            if (blockIdx.x == 0) atomicOr(p.status, kDevBadOffsets);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = *bad ? 0 : ipre[E];

    if (warp < 4) {
        const int lane = threadIdx.x & 31;
        if (warp == 0 && lane < 2) mx_producer_b<MODE>(&tmB0, &tmB1, p, seg, ipre, total, sbase, bars, abort, lane);
        else if (warp == 3 && lane < 2) mx_producer_a(&tmA, p, seg, ipre, total, sbase, bars, abort, lane);
        else if (warp == 1 && lane == 0) mx_mma(p, seg, ipre, total, sbase, bars, tmem, abort);
        if (warp == 2) mx_sf_loader<MODE>(p, seg, ipre, total, sbase + MX_OFF_SFS, bars, abort);
    } else if (warp < 8) {
        mx_epilogue<MODE>(p, seg, ipre, total, bars, tmem, abort);
    } else {
        const int n_items = static_cast<int>(blockIdx.x) < total
                                ? (total - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                                : 0;
        mx_sf_writer(p, n_items, sbase + MX_OFF_SFS, bars, tmem, abort);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, MX_TMEM_COLS);
    }
    if (threadIdx.x == 0 && *abort) atomicOr(p.status, kDevWaitTimeout);
}

// Gather: one warp per sorted row r < P_valid copies the token's code row
// and its H/32 scale bytes into expert order, the scales K-group-major
// ([ceil(H/512)][P][16]) so that the scale loader reads 32 rows' group with
// one coalesced request.
__global__ void __launch_bounds__(256) gather_mx_kernel(const uint8_t* __restrict__ codes,
                                                        const uint8_t* __restrict__ act_scales, int H, int k,
                                                        const int32_t* __restrict__ sorted_pairs,
                                                        const int32_t* __restrict__ offsets, int E, int64_t P,
                                                        uint8_t* __restrict__ a_sorted,
                                                        uint8_t* __restrict__ sa_sorted, int* __restrict__ status)
{
    const int lane = threadIdx.x & 31;
    int64_t nvalid = offsets[E];
    if (nvalid > P || nvalid < 0) nvalid = 0;  // the GEMM reports inconsistent offsets
    const int n16 = H / 16, n4 = H / 128;     // uint4 code words, uint32 scale words
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t r = warp; r < nvalid; r += nwarps) {
        const int pair = __ldg(sorted_pairs + r);
        if (pair < 0 || pair >= P) {
            if (lane == 0) atomicOr(status, kDevBadPair);
            continue;
        }
        const int64_t t = pair / k;
        const uint4* src = reinterpret_cast<const uint4*>(codes + t * H);
        uint4* dst = reinterpret_cast<uint4*>(a_sorted + r * H);
        for (int c0 = lane; c0 < n16; c0 += 4 * 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c0 + 32 * u < n16) v[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c0 + 32 * u < n16) dst[c0 + 32 * u] = v[u];
        }
        // scale words K-group-major: group g of row r at (g * P + r) * 16
        const uint32_t* ss = reinterpret_cast<const uint32_t*>(act_scales + t * (H / 32));
        for (int c = lane; c < n4; c += 32)
            reinterpret_cast<uint32_t*>(sa_sorted + ((c >> 2) * P + r) * 16)[c & 3] = __ldg(ss + c);
    }
}

// Weight scales [E, R, K/32] -> K-group-major [E][ceil(K/512)][R][16]: one
// thread per 16-byte output word; chunks at or past K/32 are written as 127.
__global__ void __launch_bounds__(256) pack_scales_kernel(const uint8_t* __restrict__ src, int64_t E, int R, int K,
                                                          uint8_t* __restrict__ dst)
{
    const int C = K / 32;
    const int G = (K + 511) / 512;
    const int64_t n = E * G * R;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int r = static_cast<int>(i % R);
        const int64_t eg = i / R;
        const int g = static_cast<int>(eg % G);
        const int64_t e = eg / G;
        const uint8_t* row = src + (e * R + r) * C;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t v = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int c = 16 * g + 4 * q + b;
                v |= static_cast<uint32_t>(c < C ? __ldg(row + c) : 0x7F) << (8 * b);
            }
            w[q] = v;
        }
        reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <int MODE>
cudaError_t run_mx(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const MxParams& p, int grid,
                   cudaStream_t s)
{
    static std::atomic<bool> attr_done[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
        err = cudaFuncSetAttribute(grouped_mx_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   mx_smem_bytes(MX_MAX_E));
        if (err != cudaSuccess) return err;
        if (dev < 64) attr_done[dev].store(true, std::memory_order_release);
    }
    grouped_mx_kernel<MODE><<<grid, MX_THREADS, mx_smem_bytes(p.E), s>>>(a, b0, b1, p);
    return cudaGetLastError();
}

}  // namespace

int mx_scale_groups(int K) { return (K + 511) / 512; }

cudaError_t launch_pack_mx_scales(const uint8_t* src, int64_t E, int R, int K, uint8_t* dst, cudaStream_t s)
{
    const int64_t n = E * mx_scale_groups(K) * R;
    if (n == 0) return cudaSuccess;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    const int64_t want = ceil_div64(n, 256);
    const int64_t cap = static_cast<int64_t>(di.sm_count) * 8;
    pack_scales_kernel<<<static_cast<int>(want < cap ? want : cap), 256, 0, s>>>(src, E, R, K, dst);
    return cudaGetLastError();
}

size_t ffn_mx_workspace_layout(int64_t T, int H, int I, int k, size_t* off_a, size_t* off_sa, size_t* off_h,
                               size_t* off_sh)
{
    const int64_t P = T * k > 0 ? T * k : 1;
    const int64_t Ip = (static_cast<int64_t>(I) + 127) / 128 * 128;
    size_t o = 256;  // status word
    *off_a = o;
    o = align_up(o + static_cast<size_t>(P) * H, 256);
    *off_sa = o;
    o = align_up(o + static_cast<size_t>(P) * mx_scale_groups(H) * 16, 256);
    *off_h = o;
    o = align_up(o + static_cast<size_t>(P) * Ip, 256);
    *off_sh = o;
    o = align_up(o + static_cast<size_t>(P) * mx_scale_groups(static_cast<int>(Ip)) * 16, 256);
    return o;
}

namespace {
cudaError_t mx_stage_mark(const FfnMxArgs& a, int i, cudaStream_t s)
{
    if (!a.stage_events || !a.stage_events[i]) return cudaSuccess;
    return record_event(a.stage_events[i], s);
}
}  // namespace

cudaError_t launch_grouped_ffn_mx(const FfnMxArgs& a, cudaStream_t s)
{
    const int64_t P = a.T * a.k;
    if (P == 0) return cudaSuccess;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    if (di.max_smem_optin < static_cast<size_t>(mx_smem_bytes(MX_MAX_E))) return cudaErrorNotSupported;
    if (a.E > MX_MAX_E) return cudaErrorNotSupported;
    const int H = a.H, I = a.I, E = a.E;
    const int Ip = (I + 127) / 128 * 128;

    cudaError_t err = mx_stage_mark(a, 0, s);
    if (err != cudaSuccess) return err;
    // 1. gather the activation rows and their scale bytes into expert order
    // (down_only: the caller supplies the intermediate; steps 1 and 3 are skipped)
    if (!a.down_only) {
        const int64_t want = ceil_div64(P, 8);
        const int64_t cap = static_cast<int64_t>(di.sm_count) * 16;
        gather_mx_kernel<<<static_cast<int>(want < cap ? want : cap), 256, 0, s>>>(
            a.codes, a.act_scales, H, a.k, a.sorted_pairs, a.expert_offsets, E, P, a.a_sorted, a.sa_sorted, a.status);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }

    // 2. tensor maps: activations and intermediate [rows, K] with 64-row
    // boxes (two per tile); gate/up and down weights with 96-row boxes (96
    // gate + 96 up rows, or two halves of 192 down rows, per tile).  The intermediate's map is I
    // wide over rows of Ip bytes, so the padding columns of the last K block
    // read as zero.
    CUtensorMap tmA1, tmG, tmU, tmA2, tmD;
    {
        const uint64_t dA[2] = {static_cast<uint64_t>(H), static_cast<uint64_t>(P)};
        const uint64_t sA[1] = {static_cast<uint64_t>(H)};
        const uint64_t dW[3] = {static_cast<uint64_t>(H), static_cast<uint64_t>(I), static_cast<uint64_t>(E)};
        const uint64_t sW[2] = {static_cast<uint64_t>(H), static_cast<uint64_t>(I) * H};
        const uint64_t dH[2] = {static_cast<uint64_t>(I), static_cast<uint64_t>(P)};
        const uint64_t sH[1] = {static_cast<uint64_t>(Ip)};
        const uint64_t dD[3] = {static_cast<uint64_t>(I), static_cast<uint64_t>(H), static_cast<uint64_t>(E)};
        const uint64_t sD[2] = {static_cast<uint64_t>(I), static_cast<uint64_t>(H) * I};
        if (!a.down_only && (!make_tmap_u8(&tmA1, a.a_sorted, 2, dA, sA, MX_BM / 2) ||
                             !make_tmap_u8(&tmG, a.w_gate, 3, dW, sW, MX_HALF) ||
                             !make_tmap_u8(&tmU, a.w_up, 3, dW, sW, MX_HALF)))
            return cudaErrorNotSupported;
        if (!make_tmap_u8(&tmA2, a.h_codes, 2, dH, sH, MX_BM / 2) || !make_tmap_u8(&tmD, a.w_down, 3, dD, sD, MX_HALF))
            return cudaErrorNotSupported;
    }
    const int grid = di.sm_count;

    // 3. gate/up GEMM with the SiLU*up + MX requantisation epilogue
    MxParams g{};
    g.E = E;
    g.num_kb = (H + MX_BK - 1) / MX_BK;
    g.num_groups = mx_scale_groups(H);
    g.n_tiles = (I + MX_HALF - 1) / MX_HALF;
    g.P = P;
    g.offsets = a.expert_offsets;
    g.a_sf = a.sa_sorted;
    g.a_chunks = H / 32;
    g.b_sf0 = a.s_gate;
    g.b_sf1 = a.s_up;
    g.b_rows = I;
    g.b_chunks = H / 32;
    g.h_codes = a.h_codes;
    g.h_scales = a.h_scales;
    g.Ip = Ip;
    g.I = I;
    g.sorted_pairs = a.sorted_pairs;
    g.topk_w = a.topk_w;
    g.y = a.y;
    g.H = H;
    g.status = a.status;
    if ((err = mx_stage_mark(a, 1, s)) != cudaSuccess) return err;
    if (!a.down_only && (err = run_mx<0>(tmA1, tmG, tmU, g, grid, s)) != cudaSuccess) return err;

    // 4. down GEMM with the routing-weighted row epilogue
    MxParams d = g;
    d.num_kb = Ip / MX_BK;
    d.num_groups = mx_scale_groups(Ip);
    d.n_tiles = (H + MX_BN - 1) / MX_BN;
    d.a_sf = a.h_scales;
    d.a_chunks = I / 32;
    d.b_sf0 = a.s_down;
    d.b_sf1 = a.s_down;
    d.b_rows = H;
    d.b_chunks = I / 32;
    if ((err = mx_stage_mark(a, 2, s)) != cudaSuccess) return err;
    if ((err = run_mx<1>(tmA2, tmD, tmD, d, grid, s)) != cudaSuccess) return err;
    return mx_stage_mark(a, 3, s);
}

}  // namespace fp8moe
