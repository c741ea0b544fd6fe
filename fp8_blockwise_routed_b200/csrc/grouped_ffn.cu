// grouped_ffn.cu -- the expert FFN of the routed-MoE W8A8 prefill path on
// sm_100a tensor cores (tcgen05 + TMEM, operands fed by TMA).
//
// Pages: blockwise FP8 MoE with 128x128 weight scales and zero-padding of a
// non-128-divisible intermediate ("Integration for GLM-4.6-FP8 and
// performance tune on H20", gap table row 6), single-wave grid sizing (row
// 3); unclamped SiLU, W8A8 ("Full GLM-5.3 streamed FP8 GPU prefill ...",
// "Design"); whole-K accumulation without split-K, fixed member order, routed
// FP32 rows written in place, one call per prompt pass ("GLM-5.3-Flash EXL3
// on CUDA: a whole prompt pass routes its experts in one call").
//
// Launch sequence of one moe_grouped_ffn call (stream-ordered, no host sync):
//   gather   : A rows in expert order: a_sorted[r] = codes[token(r)],
//              sa_sorted[r] = act_scales[token(r)]             (HBM/L2-bound)
//   gate/up  : persistent grouped GEMM, tile = 128 pair rows x (128 gate +
//              128 up) columns, one MMA of N=256 per 32-wide K step; epilogue
//              h = SiLU(g)*u, requantised per 128-group -> h codes/scales
//   down     : same kernel, tile = 128 rows x 256 output columns over the
//              intermediate; epilogue y[pair] = w_pair * o, each 256-byte row
//              segment staged in shared memory and written by a bulk copy
//              (3 weight stages; the rest of the ring holds the staging)
//
// Block scales (FP32, not powers of two) have no tensor-core path, so every
// 128-deep K block is its own MMA chain into a fresh TMEM accumulator
// ("partial"), and the epilogue warps fold it into FP32 registers with
//   acc += (sa[row,kb] * sw[nblock,kb]) * partial.
// Two partial buffers of 256 TMEM columns alternate, so the MMA of block kb+1
// overlaps the promotion of block kb.
//
// Warp roles (384 threads, one CTA per SM, grid = #SMs, static round-robin
// over work items ordered expert-major, then n-tile, then m-tile so that the
// m-tiles sharing a weight panel run at the same time and share it in L2):
//   warp 0      weight TMA producer (one lane): 2x128x128 B per stage,
//               B_STAGES deep, mbarrier complete_tx
//   warp 3      activation TMA producer (one lane): 128x128 B per stage,
//               A_STAGES deep
//   warps 1, 2  MMA issuers (one lane each; warp 1 also allocates TMEM):
//               warp 1 issues the even K blocks, warp 2 the odd ones.  A
//               thread that issues tcgen05.mma is held while the tensor pipe
//               works through it, so with one issuer the waits for the next
//               block's operands and buffer could not overlap the MMAs of
//               the current one; with two, each waits while the other's run.
//   warps 4..11 promotion + epilogue; warp w reads TMEM lanes 32*(w%4) (its
//               rows); warps 4..7 own columns [0,64) of each 128-half, warps
//               8..11 columns [64,128)
// Every wait is bounded (2 s of global time); on expiry the CTA raises an
// abort flag, records MOE_DEV_WAIT_TIMEOUT, drains and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cfloat>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace fp8moe {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 128;
constexpr int A_STAGES = 3;               // activation tiles: L2 hits, short latency
constexpr int B_STAGES = 5;               // weight tiles (gate/up): streamed from HBM, long latency
constexpr int B_STAGES_DOWN = 3;          // weight tiles (down): the rest of the ring stages y rows
constexpr int A_TILE = BM * BK;           // 16 KiB
constexpr int B_HALF = 128 * BK;          // 16 KiB
constexpr int B_TILE = 2 * B_HALF;        // 32 KiB
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 128 + EPI_WARPS * 32;  // 3 warpgroups
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64,512);
// the producer/MMA warpgroup drops to 40 and the two epilogue warpgroups rise
// to 232: 128 x 40 + 256 x 232 = 64,512, the launch total.  Each SM
// sub-partition holds one warp of each warpgroup:
// 32 x (40 + 232 + 232) = 16,128 <= 16,384 registers.
constexpr uint32_t REGS_CTRL = 40;
constexpr uint32_t REGS_EPI = 232;
static_assert(128 * REGS_CTRL + 256 * REGS_EPI <= THREADS * 168, "register split exceeds the launch budget");
static_assert(32 * (REGS_CTRL + 2 * REGS_EPI) <= 16384, "register split exceeds a sub-partition");
constexpr uint32_t TMEM_COLS = 512;       // two accumulator buffers of 256 FP32 columns
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr int MAX_E = 1024;

// shared memory map (offsets from a 1024-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + A_STAGES * A_TILE;
// down: each epilogue thread stages its 64-column y segment (256 B) here for
// a bulk copy to global memory; slots 272 B apart so a warp's 16-byte shared
// stores spread over all banks
constexpr int STAGE_SLOT = 272;
constexpr int OFF_STAGE = OFF_B + B_STAGES_DOWN * B_TILE;
constexpr int STAGE_BYTES = EPI_WARPS * 32 * STAGE_SLOT;
constexpr int RING_BYTES =
    B_STAGES * B_TILE > B_STAGES_DOWN * B_TILE + STAGE_BYTES ? B_STAGES * B_TILE : B_STAGES_DOWN * B_TILE + STAGE_BYTES;
constexpr int OFF_BARS = OFF_B + RING_BYTES;
template <int MODE>
constexpr int b_stages() { return MODE == 0 ? B_STAGES : B_STAGES_DOWN; }
// barriers: fullA, emptyA, fullB, emptyB, tfull[2], tempty[2], xbar[4]
constexpr int BAR_FULL_A = 0;
constexpr int BAR_EMPTY_A = BAR_FULL_A + A_STAGES;
constexpr int BAR_FULL_B = BAR_EMPTY_A + A_STAGES;
constexpr int BAR_EMPTY_B = BAR_FULL_B + B_STAGES;
constexpr int BAR_TFULL = BAR_EMPTY_B + B_STAGES;
constexpr int BAR_TEMPTY = BAR_TFULL + 2;
constexpr int BAR_XCHG = BAR_TEMPTY + 2;
constexpr int N_BARS = BAR_XCHG + 4;
constexpr int OFF_MISC = OFF_BARS + N_BARS * 8;
constexpr int OFF_AMAX = OFF_MISC + 16;                  // [2 parity][2 half][128 rows] floats
constexpr int OFF_SEG = OFF_AMAX + 2 * 2 * 128 * 4;      // [E+1] ints, then [E+1] ints (item prefix)
static_assert(OFF_A % 1024 == 0 && OFF_B % 1024 == 0 && A_TILE % 1024 == 0 && B_TILE % 1024 == 0,
              "128-byte-swizzled tiles need 1024-byte alignment");

// dynamic shared memory for E experts (plus slack to align the base)
constexpr int smem_bytes_for(int E) { return OFF_SEG + 2 * (E + 1) * 4 + 1024; }

struct GemmParams {
    int E;
    int rev;               // walk experts last to first (their activation rows were gathered last)
    int num_kb;            // K blocks of 128
    int n_tiles;           // output tiles per expert along N
    int64_t P;             // rows of the pair buffers (T * top_k)
    const int32_t* offsets;
    const float* a_scales; // [P, num_kb] in expert order
    const float* b_s0;     // gate/up: s_gate; down: s_down
    const float* b_s1;     // gate/up: s_up;   down: s_down
    int b_nblocks;         // scale n-blocks per expert (ceil(I/128) or H/128)
    // gate/up epilogue
    uint8_t* h_codes;      // [P, Ip]
    float* h_scales;       // [P, GI]
    int Ip;
    int GI;
    // down epilogue
    const int32_t* sorted_pairs;
    const float* topk_w;
    float* y;              // [P, H], or [y_nrows, H] rows through y_rows
    const int32_t* y_rows; // nullable: y row of each pair (-1: not written)
    int64_t y_nrows;
    int H;
    int* status;
    // combine fused into the down epilogue (MODE 2; items n-tile-major)
    float rs;
    float* out;                 // [T, H] FP32
    uint16_t* out_bf16;         // nullable
    int* cnt;                   // [T, n_tiles, 2] arrivals per token, n-tile and column half
    const int32_t* topk_ids;    // [T, k]
    const int32_t* nvalid;      // [T] valid slots per token
    int k;
};

__device__ __forceinline__ int find_expert(const int* ipre, int E, int item)
{
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ipre[mid] <= item) lo = mid;
        else hi = mid;
    }
    return lo;
}

struct Item {
    int e, nt, mt;
};

// Work items are ordered expert-major, then n-tile, then m-tile, so that the
// m-tiles sharing a weight panel are processed at the same time by
// neighbouring CTAs and share it in L2.
template <bool NTMAJOR>
__device__ __forceinline__ Item decode_item(const int* seg, const int* ipre, int E, int item, int rev)
{
    Item it;
    if (NTMAJOR) {  // n-tile-major: all m-tiles of every expert for one n-tile, then the next n-tile
        const int mt_total = ipre[E];
        it.nt = item / mt_total;
        const int local = item - it.nt * mt_total;
        const int o = find_expert(ipre, E, local);
        it.e = rev ? E - 1 - o : o;
        it.mt = local - ipre[o];
        return it;
    }
    const int o = find_expert(ipre, E, item);  // position of the expert in the walk order
    it.e = rev ? E - 1 - o : o;
    const int local = item - ipre[o];
    const int mts = (seg[it.e + 1] - seg[it.e] + BM - 1) / BM;
    it.nt = local / mts;
    it.mt = local - it.nt * mts;
    return it;
}

// A gate/up tile whose valid rows fit in 64: it takes the M = 64 path.
__device__ __forceinline__ bool small_tile(const int* seg, const Item& w)
{
    return seg[w.e + 1] - (seg[w.e] + w.mt * BM) <= 64;
}

// ---------------------------------------------------------------- roles

// Weight producer (one lane): the two 128-row weight boxes of every K block
// into a B_STAGES-deep ring.
template <int MODE>
__device__ __forceinline__ void producer_b(const CUtensorMap* tmB0, const CUtensorMap* tmB1, const GemmParams& p,
                                           const int* seg, const int* ipre, int total_items, uint32_t sbase,
                                           uint32_t bars, volatile int* abort)
{
    constexpr int BS = b_stages<MODE>();
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        const Item w = decode_item<MODE == 2>(seg, ipre, p.E, item, p.rev);
        const int n0 = (MODE == 0) ? w.nt * 128 : w.nt * 256;
        const int n1 = (MODE == 0) ? w.nt * 128 : w.nt * 256 + 128;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const int s = it % BS;
            if (!mbar_wait_bounded(bars + 8 * (BAR_EMPTY_B + s), ((it / BS) & 1) ^ 1, abort, WAIT_NS)) {
                ok = false;
                break;
            }
            const uint32_t fb = bars + 8 * (BAR_FULL_B + s);
            mbar_arrive_expect_tx(fb, B_TILE);
            const uint32_t dst = sbase + OFF_B + s * B_TILE;
            tma_load_3d(dst, tmB0, kb * BK, n0, w.e, fb);
            tma_load_3d(dst + B_HALF, tmB1, kb * BK, n1, w.e, fb);
        }
    }
    if (!ok) {  // let the copies already issued land before the CTA can exit
        for (int j = it - BS > 0 ? it - BS : 0; j < it; ++j) {
            volatile int no_abort = 0;
            mbar_wait_bounded(bars + 8 * (BAR_FULL_B + j % BS), (j / BS) & 1, &no_abort, WAIT_NS / 4);
        }
    }
}

// Activation producer (one lane): the 128-row A tile of every K block into
// an A_STAGES-deep ring.
template <int MODE>
__device__ __forceinline__ void producer_a(const CUtensorMap* tmA, const GemmParams& p, const int* seg,
                                           const int* ipre, int total_items, uint32_t sbase, uint32_t bars,
                                           volatile int* abort)
{
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        const Item w = decode_item<MODE == 2>(seg, ipre, p.E, item, p.rev);
        const int row0 = seg[w.e] + w.mt * BM;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const int s = it % A_STAGES;
            if (!mbar_wait_bounded(bars + 8 * (BAR_EMPTY_A + s), ((it / A_STAGES) & 1) ^ 1, abort, WAIT_NS)) {
                ok = false;
                break;
            }
            const uint32_t fb = bars + 8 * (BAR_FULL_A + s);
            mbar_arrive_expect_tx(fb, A_TILE);
            tma_load_2d(sbase + OFF_A + s * A_TILE, tmA, kb * BK, row0, fb);
        }
    }
    if (!ok) {
        for (int j = it - A_STAGES > 0 ? it - A_STAGES : 0; j < it; ++j) {
            volatile int no_abort = 0;
            mbar_wait_bounded(bars + 8 * (BAR_FULL_A + j % A_STAGES), (j / A_STAGES) & 1, &no_abort, WAIT_NS / 4);
        }
    }
}

// MMA issuer (one lane; two issuers split the K blocks by it%2 == parity, so
// issuer `parity` always fills accumulator buffer `parity`): per K block,
// four N=256 K=32 MMAs into the buffer (a fresh accumulation: each 128-deep K
// block is promoted with its own scales), then commits that free the A and B
// stages and hand the buffer to the epilogue.  A commit tracks the MMAs of
// the issuing thread only, which are exactly the ones it hands over.
// In the SMALL instantiation, tiles with at most 64 valid rows (gate/up and
// down, not the fused combine) use M = 64 MMAs (the accumulator then sits in
// lanes 0-15 of each 32-lane quarter), which halves the promotion work of
// their epilogue.
template <int MODE, bool SMALL>
__device__ __forceinline__ void mma_role(const GemmParams& p, const int* seg, const int* ipre, int total_items,
                                         uint32_t sbase, uint32_t bars, uint32_t tmem, volatile int* abort,
                                         int parity)
{
    constexpr int BS = b_stages<MODE>();
    constexpr uint32_t idesc128 = idesc_e4m3_f32(128, 256);
    constexpr uint32_t idesc64 = idesc_e4m3_f32(64, 256);
    int it = 0;
    int last_commit = -1;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
        uint32_t idesc = idesc128;
        if (SMALL && MODE != 2 && small_tile(seg, decode_item<false>(seg, ipre, p.E, item, p.rev))) idesc = idesc64;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            if ((it & 1) != parity) continue;  // the other issuer's K block
            const int sa = it % A_STAGES, sb = it % BS, b = it & 1;
            // no tcgen05 fence after the TMEM wait: the epilogue released the
            // buffer only after tcgen05.wait::ld, so its reads are complete
            if (!mbar_spin_bounded(bars + 8 * (BAR_TEMPTY + b), ((it >> 1) & 1) ^ 1, abort, WAIT_NS) ||
                !mbar_spin_bounded(bars + 8 * (BAR_FULL_B + sb), (it / BS) & 1, abort, WAIT_NS) ||
                !mbar_spin_bounded(bars + 8 * (BAR_FULL_A + sa), (it / A_STAGES) & 1, abort, WAIT_NS))
                goto drain;
            {
                const uint32_t a_addr = sbase + OFF_A + sa * A_TILE;
                const uint32_t b_addr = sbase + OFF_B + sb * B_TILE;
                const uint32_t d = tmem + b * 256;
#pragma unroll
                for (int kk = 0; kk < BK / 32; ++kk)
                    mma_f8(d, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                           kk > 0 ? 1u : 0u);
                mma_commit(bars + 8 * (BAR_EMPTY_A + sa));
                mma_commit(bars + 8 * (BAR_EMPTY_B + sb));
                mma_commit(bars + 8 * (BAR_TFULL + b));
                last_commit = it;
            }
        }
    }
    return;
drain:
    // wait for the MMAs already issued before TMEM is released
    if (last_commit >= 0) {
        volatile int no_abort = 0;
        mbar_wait_bounded(bars + 8 * (BAR_TFULL + (last_commit & 1)), (last_commit >> 1) & 1, &no_abort,
                          WAIT_NS / 4);
    }
}

// Gate/up epilogue of an M = 64 tile (layout above): h = SiLU(g) * u, the
// 1x128 group quantiser of each row (the row's 128 columns sit in 4 lanes of
// this warp and 4 of the partner warp of the other column half), codes
// stored two at a time.  Same arithmetic per value as the 128-row path.
__device__ __forceinline__ void small_tail(const GemmParams& p, const Item& w, int q, int half, int lane, int gA,
                                           int gB, int row_end, float (&acc0)[64], float (&acc1)[64],
                                           float* amax_x, int nitem, uint32_t xbar0, volatile int* abort)
{
    float amA = 0.f, amB = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float g = acc0[i];
        const float e = ex2_approx_ftz(-g * 1.4426950408889634f);
        const float h = (g * rcp_approx_ftz(1.0f + e)) * acc1[i];
        acc0[i] = h;
        if (i & 2) amB = fmax_nan(amB, fabsf(h));
        else amA = fmax_nan(amA, fabsf(h));
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        amA = fmax_nan(amA, __shfl_xor_sync(0xFFFFFFFFu, amA, off));
        amB = fmax_nan(amB, __shfl_xor_sync(0xFFFFFFFFu, amB, off));
    }
    const int rA = 16 * q + (lane >> 2), rB = rA + 8;
    const int par = nitem & 1;
    if ((lane & 3) == 0) {
        amax_x[(par * 2 + half) * 128 + rA] = amA;
        amax_x[(par * 2 + half) * 128 + rB] = amB;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(xbar0 + 8 * q);
    if (!__all_sync(0xFFFFFFFFu, mbar_spin_bounded(xbar0 + 8 * q, static_cast<uint32_t>(nitem & 1), abort, WAIT_NS)))
        return;
    const float oA = amax_x[(par * 2 + (half ^ 1)) * 128 + rA];
    const float oB = amax_x[(par * 2 + (half ^ 1)) * 128 + rB];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int grow = rr ? gB : gA;
        if (grow >= row_end) continue;
        const float am = rr ? amB : amA, ot = rr ? oB : oA;
        const bool nonfinite = !isfinite(am) || !isfinite(ot);
        float s = __fdiv_rn(fmaxf(am, ot), 448.0f);
        if (s == 0.f) s = 1.f;
        uint16_t* dst = reinterpret_cast<uint16_t*>(p.h_codes + static_cast<int64_t>(grow) * p.Ip + w.nt * 128 +
                                                    half * 64 + 2 * (lane & 3));
        if (nonfinite) {
            s = __int_as_float(0x7FC00000);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[4 * i] = 0x7F7F;
        } else {
            const float inv = __frcp_rn(s);
            const bool div = !isfinite(inv);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float x0 = acc0[4 * i + 2 * rr], x1 = acc0[4 * i + 2 * rr + 1];
                const float q0 = div ? __fdiv_rn(x0, s) : x0 * inv;
                const float q1 = div ? __fdiv_rn(x1, s) : x1 * inv;
                dst[4 * i] = static_cast<uint16_t>(e4m3x2(q0, q1));
            }
        }
        if (half == 0 && (lane & 3) == 0) p.h_scales[static_cast<int64_t>(grow) * p.GI + w.nt] = s;
    }
}

// Down epilogue of an M = 64 tile (layout above): y[pair] = w_pair * o for
// the thread's two rows.  The warp's 16 rows x 2 column segments (256 bytes
// each) fill its 32 staging slots exactly, so each lane then sends one
// segment by a bulk copy and no copy waits for another's read.
__device__ __forceinline__ void small_down_tail(const GemmParams& p, const Item& w, int half, int lane, int gA,
                                                int gB, int row_end, const float (&acc0)[64],
                                                const float (&acc1)[64], uint32_t warp_slots)
{
    int yA = -1, yB = -1;
    float wA = 0.f, wB = 0.f;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int g = rr ? gB : gA;
        if (g >= row_end) continue;
        const int pair = __ldg(p.sorted_pairs + g);
        int64_t yrow = -1;
        float wt = 0.f;
        if (pair >= 0 && pair < p.P) {
            wt = __ldg(p.topk_w + pair);
            yrow = p.y_rows ? __ldg(p.y_rows + pair) : pair;
        }
        if (pair < 0 || pair >= p.P || yrow >= p.y_nrows) {
            atomicOr(p.status, kDevBadPair);
            continue;
        }
        if (rr) {
            yB = static_cast<int>(yrow);
            wB = wt;
        } else {
            yA = static_cast<int>(yrow);
            wA = wt;
        }
    }
    // every slot of this warp has been read by the copies sent from it before
    bulk_wait_read_all();
    __syncwarp();
    const int rA = lane >> 2, rB = rA + 8;  // rows within the warp's 16
#pragma unroll
    for (int sgm = 0; sgm < 2; ++sgm) {
        const float* a = sgm ? acc1 : acc0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t off = (8 * i + 2 * (lane & 3)) * 4;
            st_shared_v2(warp_slots + (sgm * 16 + rA) * STAGE_SLOT + off, wA * a[4 * i], wA * a[4 * i + 1]);
            st_shared_v2(warp_slots + (sgm * 16 + rB) * STAGE_SLOT + off, wB * a[4 * i + 2], wB * a[4 * i + 3]);
        }
    }
    fence_proxy_async_smem();
    __syncwarp();
    // lane L sends segment L/16 of row L%16; that row's y row comes from the
    // lane holding it (4 * (row % 8), its first or second row)
    const int sgm = lane >> 4, row = lane & 15;
    const int src = 4 * (row & 7);
    const int ya = __shfl_sync(0xFFFFFFFFu, yA, src);
    const int yb = __shfl_sync(0xFFFFFFFFu, yB, src);
    const int yrow = row < 8 ? ya : yb;
    const int c = w.nt * 256 + sgm * 128 + half * 64;
    if (yrow >= 0 && c < p.H)
        bulk_store(p.y + static_cast<int64_t>(yrow) * p.H + c, warp_slots + (sgm * 16 + row) * STAGE_SLOT, 256);
    bulk_commit();
}

template <int MODE, bool SMALL>
__device__ __forceinline__ void epilogue_role(const GemmParams& p, const int* seg, const int* ipre, int total_items, uint32_t bars,
                              uint32_t tmem, float* amax_x, volatile int* abort)
{
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - 4) >> 2;        // column half-slice of each 128-wide half
    const int trow = q * 32 + lane;          // row within the tile
    const uint32_t tfull0 = bars + 8 * BAR_TFULL, tempty0 = bars + 8 * BAR_TEMPTY, xbar0 = bars + 8 * BAR_XCHG;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int it = 0;
    int nitem = 0;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x, ++nitem) {
        const Item w = decode_item<MODE == 2>(seg, ipre, p.E, item, p.rev);
        const int r = seg[w.e] + w.mt * BM + trow;
        const bool valid = r < seg[w.e + 1];
        const int64_t ra = r < p.P ? r : p.P - 1;
        const float* sa_row = p.a_scales + ra * p.num_kb;
        int nb0, nb1;
        if (MODE == 0) {
            nb0 = nb1 = w.nt;
        } else {
            nb0 = 2 * w.nt;
            nb1 = 2 * w.nt + 1;
        }
        const float* s0 = p.b_s0 + (static_cast<int64_t>(w.e) * p.b_nblocks + nb0) * p.num_kb;
        const float* s1 = p.b_s1 + (static_cast<int64_t>(w.e) * p.b_nblocks + (nb1 < p.b_nblocks ? nb1 : nb0)) * p.num_kb;
        const bool has1 = nb1 < p.b_nblocks;
        // down: the row's pair index and routing weight, fetched before the
        // K loop so that the tail does not wait on them
        int pair = -1;
        int64_t yrow = -1;
        float wt = 0.f;
        if (MODE != 0 && valid) {
            pair = __ldg(p.sorted_pairs + r);
            if (pair >= 0 && pair < p.P) {
                wt = __ldg(p.topk_w + pair);
                yrow = p.y_rows ? __ldg(p.y_rows + pair) : pair;
            }
        }
        int nval = 0;  // fused combine: valid slots of this row's token
        if (MODE == 2 && pair >= 0 && pair < p.P) nval = __ldg(p.nvalid + pair / p.k);

        float acc0[64], acc1[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            acc0[i] = 0.f;
            acc1[i] = 0.f;
        }
        if (SMALL && MODE != 2 && small_tile(seg, w)) {
            // M = 64 tile: rows 16q + j/4 ... live in lanes 0-15 of quarter q.
            // This thread holds rows rA = 16q + lane/4 and rB = rA + 8, 16
            // columns of each 128-column half (its 64 columns, 2 per 8-column
            // group): acc0[4i + e] / acc1[4i + e], e < 2 row rA, e >= 2 row
            // rB, columns half*64 + 8i + 2(lane%4) + (e&1) of each half.
            const int gA = seg[w.e] + w.mt * BM + 16 * q + (lane >> 2), gB = gA + 8;
            const float* saA = p.a_scales + static_cast<int64_t>(gA < p.P ? gA : p.P - 1) * p.num_kb;
            const float* saB = p.a_scales + static_cast<int64_t>(gB < p.P ? gB : p.P - 1) * p.num_kb;
            const int sb0 = MODE == 0 ? w.nt : 2 * w.nt;
            const int sb1 = MODE == 0 ? w.nt : 2 * w.nt + 1;
            const bool two = sb1 < p.b_nblocks;
            const float* s0 = p.b_s0 + (static_cast<int64_t>(w.e) * p.b_nblocks + sb0) * p.num_kb;
            const float* s1 = p.b_s1 + (static_cast<int64_t>(w.e) * p.b_nblocks + (two ? sb1 : sb0)) * p.num_kb;
            float aA_n = __ldg(saA), aB_n = __ldg(saB), w0_n = __ldg(s0), w1_n = two ? __ldg(s1) : 0.f;
            for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                const float c0A = aA_n * w0_n, c0B = aB_n * w0_n;
                const float c1A = aA_n * w1_n, c1B = aB_n * w1_n;
                if (kb + 1 < p.num_kb) {
                    aA_n = __ldg(saA + kb + 1);
                    aB_n = __ldg(saB + kb + 1);
                    w0_n = __ldg(s0 + kb + 1);
                    if (two) w1_n = __ldg(s1 + kb + 1);
                }
                const int b = it & 1;
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(tfull0 + 8 * b, (it >> 1) & 1, abort, WAIT_NS)))
                    return;
                const uint32_t col = lane_base + b * 256 + half * 64;
                uint32_t ra[32], rb[32];
                tmem_ld16x256_x8_issue(col, ra);        // gate columns
                tmem_ld_wait(ra);
                tmem_ld16x256_x8_issue(col + 128, rb);  // up columns
#pragma unroll
                for (int i = 0; i < 32; ++i) acc0[i] = fmaf((i & 2) ? c0B : c0A, __uint_as_float(ra[i]), acc0[i]);
                tmem_ld_wait(rb);
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty0 + 8 * b);
#pragma unroll
                for (int i = 0; i < 32; ++i) acc1[i] = fmaf((i & 2) ? c1B : c1A, __uint_as_float(rb[i]), acc1[i]);
            }
            if (MODE == 0)
                small_tail(p, w, q, half, lane, gA, gB, seg[w.e + 1], acc0, acc1, amax_x, nitem, xbar0, abort);
            else
                small_down_tail(p, w, half, lane, gA, gB, seg[w.e + 1], acc0, acc1,
                                bars - OFF_BARS + OFF_STAGE + (warp - 4) * 32 * STAGE_SLOT);
            continue;
        }
        // scales of K block kb+1 are fetched while block kb is promoted
        float sa_n = __ldg(sa_row), w0_n = __ldg(s0), w1_n = has1 ? __ldg(s1) : 0.f;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const float c0 = sa_n * w0_n;
            const float c1 = sa_n * w1_n;
            if (kb + 1 < p.num_kb) {
                sa_n = __ldg(sa_row + kb + 1);
                w0_n = __ldg(s0 + kb + 1);
                if (has1) w1_n = __ldg(s1 + kb + 1);
            }
            // buffer it%2 holds the partial of this K block: columns [0,128)
            // -> acc0 (gate / first output block), [128,256) -> acc1; this
            // thread reads its 64 columns of each half in 32-column loads,
            // each load overlapping the FMAs of the one before, and releases
            // the buffer as soon as the last load has landed
            const int b = it & 1;
            // a suspending wait: the epilogue warps share their sub-partitions
            // with the producer and issuer lanes, which a polling loop would
            // take issue slots from
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(tfull0 + 8 * b, (it >> 1) & 1, abort, WAIT_NS))) return;
            const uint32_t col = lane_base + b * 256 + half * 64;
            uint32_t ra[32], rb[32];
            tmem_ld32_issue(col, ra);
            tmem_ld_wait(ra);
            tmem_ld32_issue(col + 32, rb);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc0[i] = fmaf(c0, __uint_as_float(ra[i]), acc0[i]);
            tmem_ld_wait(rb);
            tmem_ld32_issue(col + 128, ra);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc0[32 + i] = fmaf(c0, __uint_as_float(rb[i]), acc0[32 + i]);
            tmem_ld_wait(ra);
            tmem_ld32_issue(col + 160, rb);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc1[i] = fmaf(c1, __uint_as_float(ra[i]), acc1[i]);
            tmem_ld_wait(rb);
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty0 + 8 * b);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc1[32 + i] = fmaf(c1, __uint_as_float(rb[i]), acc1[32 + i]);
        }

        if (MODE == 0) {
            // h = SiLU(g) * u (unclamped), then the 1x128 group quantiser over
            // this row's 128 intermediate columns [nt*128, nt*128+128), half of
            // which this thread holds; the other half comes through shared
            // memory from the partner warp of the same lane quarter.
            // amax is NaN-propagating, so it is finite exactly when every h
            // of this half-row is
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float g = acc0[i];
                // SiLU(g) = g / (1 + e^-g), e^-g = 2^(-g log2 e), with the
                // hardware exp2 and reciprocal approximations (a few ulp; the
                // requantisation below is insensitive to that except within
                // it of a rounding boundary).  e^-g overflows to +inf for
                // g < -88.7, where the reciprocal gives 0 and h = -0 * u.
                const float e = ex2_approx_ftz(-g * 1.4426950408889634f);
                const float h = (g * rcp_approx_ftz(1.0f + e)) * acc1[i];
                acc0[i] = h;
                amax = fmax_nan(amax, fabsf(h));
            }
            const int par = nitem & 1;
            amax_x[(par * 2 + half) * 128 + trow] = amax;
            __syncwarp();
            if (lane == 0) mbar_arrive(xbar0 + 8 * q);
            if (!__all_sync(0xFFFFFFFFu,
                            mbar_spin_bounded(xbar0 + 8 * q, static_cast<uint32_t>(nitem & 1), abort, WAIT_NS)))
                return;
            const float other = amax_x[(par * 2 + (half ^ 1)) * 128 + trow];
            const bool nonfinite = !isfinite(amax) || !isfinite(other);
            float s = __fdiv_rn(fmaxf(amax, other), 448.0f);
            if (s == 0.f) s = 1.f;
            if (valid) {
                uint8_t* dst = p.h_codes + static_cast<int64_t>(r) * p.Ip + w.nt * 128 + half * 64;
                if (nonfinite) {
                    s = __int_as_float(0x7FC00000);
                    const uint4 nanq = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
#pragma unroll
                    for (int c = 0; c < 4; ++c) reinterpret_cast<uint4*>(dst)[c] = nanq;
                } else {
                    // h / s as h times the correctly rounded reciprocal of s
                    // (within 1 ulp of the quotient; a code can differ from
                    // the divide's only when h/s lies within that ulp of an
                    // E4M3 rounding boundary).  Scales whose reciprocal
                    // overflows use the divide.
                    const float inv = __frcp_rn(s);
                    if (!isfinite(inv)) {  // rare: divide each value
#pragma unroll
                        for (int i = 0; i < 64; ++i) acc0[i] = __fdiv_rn(acc0[i], s);
                    } else {
#pragma unroll
                        for (int i = 0; i < 64; ++i) acc0[i] *= inv;
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t wv[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int i = c * 16 + j * 4;
                            wv[j] = e4m3x2(acc0[i], acc0[i + 1]) | (e4m3x2(acc0[i + 2], acc0[i + 3]) << 16);
                        }
                        reinterpret_cast<uint4*>(dst)[c] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    }
                }
                if (half == 0) p.h_scales[static_cast<int64_t>(r) * p.GI + w.nt] = s;
            }
        } else if (MODE == 2) {
            // Combine fused into the epilogue.  The row's two 64-column y
            // segments are written, made visible, and counted on the
            // (token, n-tile, column half) arrival counter; the thread whose
            // arrival completes the token's valid slots marks that segment
            // pair ready, and the whole warp then sums each ready token's
            // slot rows in slot order (the combine's arithmetic: from zero,
            // valid slots in order, times routed_scaling) with coalesced
            // loads.  The order of arrival does not change any bit.
            const bool mine = valid && pair >= 0 && pair < p.P;
            if (valid && !mine) atomicOr(p.status, kDevBadPair);
            const int c0 = w.nt * 256 + half * 64;
            const int c1 = c0 + 128;
            if (mine) {
                float* dst = p.y + static_cast<int64_t>(pair) * p.H;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int c = hh ? c1 : c0;
                    if (c >= p.H) continue;
                    const float* a = hh ? acc1 : acc0;
                    float4* g = reinterpret_cast<float4*>(dst + c);
#pragma unroll
                    for (int q4 = 0; q4 < 16; ++q4)
                        g[q4] = make_float4(wt * a[4 * q4], wt * a[4 * q4 + 1], wt * a[4 * q4 + 2], wt * a[4 * q4 + 3]);
                }
            }
            __threadfence();
            const int tok = mine ? pair / p.k : 0;
            bool last = false;
            if (mine) last = atomicAdd(p.cnt + (static_cast<int64_t>(tok) * p.n_tiles + w.nt) * 2 + half, 1) == nval - 1;
            uint32_t ready = __ballot_sync(0xFFFFFFFFu, last);
            if (ready) __threadfence();
            while (ready) {
                const int L = __ffs(ready) - 1;
                ready &= ready - 1;
                const int64_t t = __shfl_sync(0xFFFFFFFFu, tok, L);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int c = (hh ? c1 : c0) + 2 * lane;  // this lane's two columns
                    if ((hh ? c1 : c0) >= p.H) continue;
                    float2 acc = make_float2(0.f, 0.f);
                    for (int j0 = 0; j0 < p.k; j0 += 8) {
                        float2 v[8];
                        bool ok[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int j = j0 + u;
                            const int e = (j < p.k) ? __ldg(p.topk_ids + t * p.k + j) : -1;
                            ok[u] = e >= 0 && e < p.E;
                            v[u] = ok[u] ? __ldcg(reinterpret_cast<const float2*>(p.y + (t * p.k + j) * p.H + c))
                                         : make_float2(0.f, 0.f);
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            if (!ok[u]) continue;
                            acc.x += v[u].x;
                            acc.y += v[u].y;
                        }
                    }
                    const float2 o = make_float2(p.rs * acc.x, p.rs * acc.y);
                    *reinterpret_cast<float2*>(p.out + t * p.H + c) = o;
                    if (p.out_bf16) {
                        const __nv_bfloat162 bb = __floats2bfloat162_rn(o.x, o.y);
                        *reinterpret_cast<__nv_bfloat162*>(p.out_bf16 + t * p.H + c) = bb;
                    }
                }
            }
        } else {
            if (valid) {
                if (pair < 0 || pair >= p.P || yrow >= p.y_nrows) {
                    atomicOr(p.status, kDevBadPair);
                } else if (yrow >= 0) {
                    float* dst = p.y + yrow * p.H;
                    const int c0 = w.nt * 256 + half * 64;
                    const int c1 = c0 + 128;
                    // Each 64-column segment (256 contiguous bytes of the
                    // pair's y row) goes through this thread's shared slot
                    // to a bulk copy, so the TMA engine does the global
                    // writes while the warp returns to the next item.  The
                    // slot is rewritten only after the copies that read it
                    // have done so.
                    const uint32_t slot = bars - OFF_BARS + OFF_STAGE + (threadIdx.x - 128) * STAGE_SLOT;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int c = hh ? c1 : c0;
                        if (c >= p.H) continue;
                        const float* a = hh ? acc1 : acc0;
                        bulk_wait_read_all();
#pragma unroll
                        for (int q4 = 0; q4 < 16; ++q4)
                            st_shared_v4(slot + 16 * q4, wt * a[4 * q4], wt * a[4 * q4 + 1], wt * a[4 * q4 + 2],
                                         wt * a[4 * q4 + 3]);
                        fence_proxy_async_smem();
                        bulk_store(dst + c, slot, 256);
                        bulk_commit();
                    }
                }
            }
        }
    }
}

template <int MODE, bool SMALL>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + OFF_BARS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
    int* bad = reinterpret_cast<int*>(smem + OFF_MISC + 8);
    float* amax_x = reinterpret_cast<float*>(smem + OFF_AMAX);
    int* seg = reinterpret_cast<int*>(smem + OFF_SEG);
    int* ipre = seg + (p.E + 1);
    const int warp = threadIdx.x >> 5;
    const int E = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < A_STAGES; ++s) {
            mbar_init(bars + 8 * (BAR_FULL_A + s), 1);   // producer arrive + tx
            mbar_init(bars + 8 * (BAR_EMPTY_A + s), 1);  // MMA commit
        }
        for (int s = 0; s < B_STAGES; ++s) {
            mbar_init(bars + 8 * (BAR_FULL_B + s), 1);
            mbar_init(bars + 8 * (BAR_EMPTY_B + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars + 8 * (BAR_TFULL + b), 1);           // MMA commit
            mbar_init(bars + 8 * (BAR_TEMPTY + b), EPI_WARPS);  // epilogue warps
        }
        for (int q = 0; q < 4; ++q) mbar_init(bars + 8 * (BAR_XCHG + q), 2);  // amax exchange
        *abort = 0;
        *bad = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && threadIdx.x == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB0);
        prefetch_tmap(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i <= E; i += blockDim.x) seg[i] = __ldg(p.offsets + i);
    __syncthreads();
    if (threadIdx.x == 0) {
        int okv = (seg[0] == 0);
        int acc = 0;
        ipre[0] = 0;
        for (int o = 0; o < E; ++o) {
            const int e = p.rev ? E - 1 - o : o;  // experts are walked in this order
            const int c = seg[e + 1] - seg[e];
            if (c < 0 || seg[e + 1] > p.P) okv = 0;
            const int mts = c > 0 ? (c + BM - 1) / BM : 0;
            acc += (MODE == 2) ? mts : mts * p.n_tiles;
            ipre[o + 1] = acc;
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
    const int total_items = *bad ? 0 : ((MODE == 2) ? ipre[E] * p.n_tiles : ipre[E]);

    if (warp < 4) {
        setmaxnreg_dec<REGS_CTRL>();
        if ((threadIdx.x & 31) == 0) {
            if (warp == 0) producer_b<MODE>(&tmB0, &tmB1, p, seg, ipre, total_items, sbase, bars, abort);
            else if (warp == 1 || warp == 2)
                mma_role<MODE, SMALL>(p, seg, ipre, total_items, sbase, bars, tmem, abort, warp - 1);
            else if (warp == 3) producer_a<MODE>(&tmA, p, seg, ipre, total_items, sbase, bars, abort);
        }
    } else {
        setmaxnreg_inc<REGS_EPI>();
        epilogue_role<MODE, SMALL>(p, seg, ipre, total_items, bars, tmem, amax_x, abort);
        // the y bulk copies must be done with shared memory (and complete)
        // before the CTA exits
        if (MODE != 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (threadIdx.x == 0 && *abort) atomicOr(p.status, kDevWaitTimeout);
}

// Gather: one warp per sorted row r < P_valid copies the token's code row
// and scale row into expert order.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint8_t* __restrict__ codes,
                                                          const float* __restrict__ act_scales, int H, int k,
                                                          const int32_t* __restrict__ sorted_pairs,
                                                          const int32_t* __restrict__ offsets, int E, int64_t P,
                                                          uint8_t* __restrict__ a_sorted,
                                                          float* __restrict__ sa_sorted, int* __restrict__ status)
{
    const int lane = threadIdx.x & 31;
    int64_t nvalid = offsets[E];
    if (nvalid > P || nvalid < 0) nvalid = 0;  // the GEMM reports inconsistent offsets
    const int GH = H / 128;
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
        // four 16-byte loads in flight per lane, then their stores
        const int n16 = H / 16;
        for (int c0 = lane; c0 < n16; c0 += 4 * 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c0 + 32 * u < n16) v[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c0 + 32 * u < n16) dst[c0 + 32 * u] = v[u];
        }
        for (int c = lane; c < GH; c += 32) sa_sorted[r * GH + c] = __ldg(act_scales + t * GH + c);
    }
}

// Fused combine, before the GEMMs: per token (one warp each), zero the
// arrival counters, count the valid slots, and write the zero row of a token
// with none (no arrival will come for it).
__global__ void __launch_bounds__(256) fuse_prep_kernel(const int32_t* __restrict__ ids, int64_t T, int k, int E,
                                                        int n_tiles, int H, int* __restrict__ cnt,
                                                        int32_t* __restrict__ nvalid, float* __restrict__ out,
                                                        uint16_t* __restrict__ out_bf16)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    for (int i = lane; i < n_tiles * 2; i += 32) cnt[t * n_tiles * 2 + i] = 0;
    int n = 0;
    for (int j = 0; j < k; ++j) {
        const int e = __ldg(ids + t * k + j);
        n += (e >= 0 && e < E) ? 1 : 0;
    }
    if (lane == 0) nvalid[t] = n;
    if (n == 0) {
        for (int c = lane; c < H; c += 32) {
            out[t * H + c] = 0.f;
            if (out_bf16) out_bf16[t * H + c] = 0;
        }
    }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Row-major uint8 tensor of `rank` dims (innermost first), tile box of
// 128 bytes x box_rows (x 1), 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               uint32_t box_rows)
{
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t gdim[3], gstr[2];
    cuuint32_t box[3], estr[3];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        estr[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) gstr[i] = strides_bytes[i];
    box[0] = 128;
    box[1] = box_rows;
    if (rank == 3) box[2] = 1;
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), gdim, gstr, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE, bool SMALL>
cudaError_t run_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const GemmParams& p,
                     int grid, cudaStream_t s)
{
    const int smem = smem_bytes_for(MAX_E);
    // per device, once; host threads may launch concurrently
    static std::atomic<bool> attr_done[64];  // one set per instantiation
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
        err = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, SMALL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err != cudaSuccess) return err;
        if (dev < 64) attr_done[dev].store(true, std::memory_order_release);
    }
    grouped_gemm_kernel<MODE, SMALL><<<grid, THREADS, smem_bytes_for(p.E), s>>>(a, b0, b1, p);
    return cudaGetLastError();
}

}  // namespace

bool make_tmap_u8(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                  uint32_t box_rows)
{
    return make_tmap(m, base, rank, dims, strides_bytes, box_rows);
}

size_t ffn_workspace_layout(int64_t T, int H, int I, int k, size_t* off_a, size_t* off_sa, size_t* off_h,
                            size_t* off_sh, size_t* off_cnt, size_t* off_nv)
{
    const int64_t P = T * k > 0 ? T * k : 1;
    const int GI = (I + 127) / 128;
    const int64_t Ip = static_cast<int64_t>(GI) * 128;
    size_t o = 256;  // status word
    *off_a = o;
    o = align_up(o + static_cast<size_t>(P) * H, 256);
    *off_sa = o;
    o = align_up(o + static_cast<size_t>(P) * (H / 128) * 4, 256);
    *off_h = o;
    o = align_up(o + static_cast<size_t>(P) * Ip, 256);
    *off_sh = o;
    o = align_up(o + static_cast<size_t>(P) * GI * 4, 256);
    // fused combine: arrival counters [T, ceil(H/256), 2], valid slots [T]
    const size_t t = static_cast<size_t>(T > 0 ? T : 1);
    if (off_cnt) *off_cnt = o;
    o = align_up(o + t * ((H + 255) / 256) * 2 * 4, 256);
    if (off_nv) *off_nv = o;
    o = align_up(o + t * 4, 256);
    return o;
}

namespace {
cudaError_t stage_mark(const FfnArgs& a, int i, cudaStream_t s)
{
    if (!a.stage_events || !a.stage_events[i]) return cudaSuccess;
    return record_event(a.stage_events[i], s);
}
}  // namespace

cudaError_t launch_grouped_ffn(const FfnArgs& a, cudaStream_t s)
{
    const int64_t P = a.T * a.k;
    if (P == 0) return cudaSuccess;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    if (di.max_smem_optin < static_cast<size_t>(smem_bytes_for(MAX_E))) return cudaErrorNotSupported;
    const int H = a.H, I = a.I, E = a.E;
    const int GH = H / 128, GI = (I + 127) / 128, Ip = GI * 128;

    cudaError_t err = stage_mark(a, 0, s);
    if (err != cudaSuccess) return err;
    // 1. gather the A operand rows (and their scales) into expert order
    // (down_only: the caller supplies the intermediate; steps 1 and 3 are skipped)
    if (!a.down_only) {
        const int64_t want = ceil_div64(P, 8);
        const int64_t cap = static_cast<int64_t>(di.sm_count) * 16;
        gather_rows_kernel<<<static_cast<int>(want < cap ? want : cap), 256, 0, s>>>(
            a.codes, a.act_scales, H, a.k, a.sorted_pairs, a.expert_offsets, E, P, a.a_sorted, a.sa_sorted,
            a.status);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }

    // 2. tensor maps
    CUtensorMap tmA1, tmG, tmU, tmA2, tmD;
    {
        const uint64_t dA[2] = {static_cast<uint64_t>(H), static_cast<uint64_t>(P)};
        const uint64_t sA[1] = {static_cast<uint64_t>(H)};
        const uint64_t dW[3] = {static_cast<uint64_t>(H), static_cast<uint64_t>(I), static_cast<uint64_t>(E)};
        const uint64_t sW[2] = {static_cast<uint64_t>(H), static_cast<uint64_t>(I) * H};
        const uint64_t dH[2] = {static_cast<uint64_t>(Ip), static_cast<uint64_t>(P)};
        const uint64_t sH[1] = {static_cast<uint64_t>(Ip)};
        const uint64_t dD[3] = {static_cast<uint64_t>(I), static_cast<uint64_t>(H), static_cast<uint64_t>(E)};
        const uint64_t sD[2] = {static_cast<uint64_t>(I), static_cast<uint64_t>(H) * I};
        if (!a.down_only && (!make_tmap(&tmA1, a.a_sorted, 2, dA, sA, 128) ||
                             !make_tmap(&tmG, a.w_gate, 3, dW, sW, 128) || !make_tmap(&tmU, a.w_up, 3, dW, sW, 128)))
            return cudaErrorNotSupported;
        if (!make_tmap(&tmA2, a.h_codes, 2, dH, sH, 128) || !make_tmap(&tmD, a.w_down, 3, dD, sD, 128))
            return cudaErrorNotSupported;
    }
    const int grid = di.sm_count;

    // 3. gate/up GEMM with the SiLU*up + requantisation epilogue
    GemmParams g{};
    g.E = E;
    g.num_kb = GH;
    g.n_tiles = GI;
    g.P = P;
    g.offsets = a.expert_offsets;
    g.a_scales = a.sa_sorted;
    g.rev = 1;
    g.b_s0 = a.s_gate;
    g.b_s1 = a.s_up;
    g.b_nblocks = GI;
    g.h_codes = a.h_codes;
    g.h_scales = a.h_scales;
    g.Ip = Ip;
    g.GI = GI;
    g.sorted_pairs = a.sorted_pairs;
    g.topk_w = a.topk_w;
    g.y = a.y;
    g.y_rows = a.y_rows;
    g.y_nrows = a.y_rows ? a.y_nrows : P;
    g.H = H;
    g.status = a.status;
    if ((err = stage_mark(a, 1, s)) != cudaSuccess) return err;
    // The M = 64 variant of the gate/up and down kernels pays off when many
    // experts receive few rows (a skewed routing of a short batch); with 256
    // or more rows per expert on average nearly every tile is full, and the
    // variant without that path is faster.  Both give identical bits.
    const bool small = P < static_cast<int64_t>(E) * 256;
    if (!a.down_only) {
        err = small ? run_gemm<0, true>(tmA1, tmG, tmU, g, grid, s) : run_gemm<0, false>(tmA1, tmG, tmU, g, grid, s);
        if (err != cudaSuccess) return err;
    }

    // 4. down GEMM with the routing-weighted row epilogue
    GemmParams d = g;
    d.num_kb = GI;
    d.n_tiles = (H + 255) / 256;
    d.a_scales = a.h_scales;
    d.b_s0 = a.s_down;
    d.b_s1 = a.s_down;
    d.b_nblocks = GH;
    d.rev = 0;
    if (a.fuse) {
        // prep (counters, valid slots, empty rows), then the down items
        // n-tile-major so that a token's slot rows meet in L2
        const int nt_down = (H + 255) / 256;
        fuse_prep_kernel<<<static_cast<int>(ceil_div64(a.T * 32, 256)), 256, 0, s>>>(
            a.topk_ids, a.T, a.k, E, nt_down, H, a.cnt, a.nvalid, a.out, a.out_bf16);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        d.rs = a.rs;
        d.out = a.out;
        d.out_bf16 = a.out_bf16;
        d.cnt = a.cnt;
        d.topk_ids = a.topk_ids;
        d.nvalid = a.nvalid;
        d.k = a.k;
    }
    if ((err = stage_mark(a, 2, s)) != cudaSuccess) return err;
    if ((err = a.fuse    ? run_gemm<2, false>(tmA2, tmD, tmD, d, grid, s)
               : small ? run_gemm<1, true>(tmA2, tmD, tmD, d, grid, s)
                       : run_gemm<1, false>(tmA2, tmD, tmD, d, grid, s)) != cudaSuccess)
        return err;
    return stage_mark(a, 3, s);
}

}  // namespace fp8moe
