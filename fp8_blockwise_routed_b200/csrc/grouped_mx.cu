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
//   gate/up  : tile 128 rows x (64 gate + 64 up) columns; epilogue
//              h = SiLU(g) * u, MX-requantised per 32 columns
//   down     : tile 128 rows x 128 output columns; epilogue y[pair] = w * o
//
// Warp roles (384 threads, one CTA per SM, persistent over work items ordered
// expert-major, then n-tile, then m-tile):
//   warp 0      weight TMA producer (one lane)
//   warp 1      MMA issuer (one lane; also allocates TMEM)
//   warp 3      activation TMA producer (one lane)
//   warps 4..7  epilogue: warp w drains TMEM lanes 32*(w%4), once per item
//   warps 8..11 scale stagers: per K block, write the tile's A and B scale
//               bytes into a TMEM ring with tcgen05.st.  The MMA reads a
//               row's scale from the lane of that row in every 32-lane
//               sub-partition, so each of the four warps writes the same
//               data into its own sub-partition.
// TMEM: two 128-column accumulators (items alternate) and SF_SLOTS slots of
// 8 scale columns.  Scale layout (K block of 128 = 4 chunks of 32): row m of
// the A tile -> lanes m%32 (+32 per sub-partition), column m/32, byte j =
// chunk j; B row n likewise in the slot's columns 4..7.  The MMA of chunk j
// selects byte j (scale-factor id j).
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
constexpr int MX_BK = 128;
constexpr int MX_STAGES = 6;
constexpr int MX_A_TILE = 128 * 128;  // 16 KiB
constexpr int MX_B_TILE = 128 * 128;  // 16 KiB
constexpr int MX_STAGE = MX_A_TILE + MX_B_TILE;
constexpr int MX_THREADS = 384;
constexpr int SF_SLOTS = 16;
constexpr int SF_COL = 256;             // scale ring starts after the two accumulators
constexpr uint32_t MX_TMEM_COLS = 512;  // 2 x 128 + 16 x 8 = 384 used
constexpr uint64_t MX_WAIT_NS = 2000000000ull;
constexpr int MX_MAX_E = 1024;

constexpr int MB_FULL = 0;                       // [stages]: both producers (arrive + tx)
constexpr int MB_EMPTY = MB_FULL + MX_STAGES;    // [stages]: MMA commit
constexpr int MB_SFF = MB_EMPTY + MX_STAGES;     // [slots]: the four stager warps
constexpr int MB_SFE = MB_SFF + SF_SLOTS;        // [slots]: MMA commit
constexpr int MB_AF = MB_SFE + SF_SLOTS;         // [2]: accumulator full (MMA commit)
constexpr int MB_AE = MB_AF + 2;                 // [2]: accumulator drained (four epilogue warps)
constexpr int MB_N = MB_AE + 2;
constexpr int MX_OFF_BARS = MX_STAGES * MX_STAGE;
constexpr int MX_OFF_MISC = MX_OFF_BARS + MB_N * 8;
constexpr int MX_OFF_SEG = MX_OFF_MISC + 16;  // [E+1] offsets, then [E+1] item prefix
constexpr int mx_smem_bytes(int E) { return MX_OFF_SEG + 2 * (E + 1) * 4 + 1024; }
static_assert(SF_COL + SF_SLOTS * 8 <= static_cast<int>(MX_TMEM_COLS), "scale ring exceeds TMEM");

struct MxParams {
    int E;
    int num_kb;            // K blocks of 128
    int n_tiles;           // output tiles per expert
    int64_t P;             // rows of the pair buffers (T * top_k)
    const int32_t* offsets;
    const uint8_t* a_sf;   // [P, a_sf_stride] scale bytes of the A rows (expert order)
    int a_sf_stride;       // bytes per A scale row
    int a_chunks;          // valid 32-column chunks of an A row (K / 32)
    const uint8_t* b_sf0;  // gate/up: s_gate; down: s_down ([E, b_rows, b_sf_stride])
    const uint8_t* b_sf1;  // gate/up: s_up
    int b_rows;            // weight rows per expert (I or H)
    int b_sf_stride;       // bytes per weight scale row (H/32 or I/32)
    int b_chunks;          // valid chunks of a weight row (K / 32)
    // gate/up epilogue
    uint8_t* h_codes;      // [P, Ip]
    uint8_t* h_scales;     // [P, Ip/32]
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

// Four scale bytes of one row for the K block starting at chunk c0 (of nvalid
// chunks); missing chunks read as 127 (2^0), so zero operands stay zero.
__device__ __forceinline__ uint32_t load_sf4(const uint8_t* row, int c0, int nvalid, bool aligned4)
{
    if (aligned4 && c0 + 4 <= nvalid) return __ldg(reinterpret_cast<const uint32_t*>(row + c0));
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t b = (c0 + j < nvalid) ? static_cast<uint32_t>(__ldg(row + c0 + j)) : 127u;
        v |= b << (8 * j);
    }
    return v;
}

// ---------------------------------------------------------------- roles

template <int MODE>
__device__ __forceinline__ void mx_producer_b(const CUtensorMap* tm0, const CUtensorMap* tm1, const MxParams& p,
                                              const int* seg, const int* ipre, int total, uint32_t sbase,
                                              uint32_t bars, volatile int* abort)
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
            mbar_arrive_expect_tx(fb, MX_B_TILE);
            const uint32_t dst = sbase + s * MX_STAGE + MX_A_TILE;
            if (MODE == 0) {  // 64 gate rows, then 64 up rows, of n-tile nt
                tma_load_3d(dst, tm0, kb * MX_BK, w.nt * 64, w.e, fb);
                tma_load_3d(dst + MX_B_TILE / 2, tm1, kb * MX_BK, w.nt * 64, w.e, fb);
            } else {
                tma_load_3d(dst, tm0, kb * MX_BK, w.nt * 128, w.e, fb);
            }
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
                                              volatile int* abort)
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
            mbar_arrive_expect_tx(fb, MX_A_TILE);
            tma_load_2d(sbase + s * MX_STAGE, tmA, kb * MX_BK, row0, fb);
        }
    }
    if (!ok) {
        for (int j = it - MX_STAGES > 0 ? it - MX_STAGES : 0; j < it; ++j) {
            volatile int no_abort = 0;
            mbar_wait_bounded(bars + 8 * (MB_FULL + j % MX_STAGES), (j / MX_STAGES) & 1, &no_abort, MX_WAIT_NS / 4);
        }
    }
}

// Scale stager (warps 8..11, all lanes): per K block, lane t of the warp on
// sub-partition q writes lane 32q + t of the slot: columns 0..3 the A scales
// of tile rows t, t+32, t+64, t+96; columns 4..7 those of B rows t .. t+96.
template <int MODE>
__device__ __forceinline__ void mx_stager(const MxParams& p, const int* seg, const int* ipre, int total,
                                          uint32_t bars, uint32_t tmem, volatile int* abort)
{
    const int lane = threadIdx.x & 31;
    const int q = (threadIdx.x >> 5) & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const bool a_aligned = (p.a_sf_stride & 3) == 0;
    const bool b_aligned = (p.b_sf_stride & 3) == 0;
    int it = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const MxItem w = mx_decode(seg, ipre, p.E, item);
        const int row0 = seg[w.e] + w.mt * MX_BM;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const int ss = it % SF_SLOTS;
            uint32_t v[8];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                int64_t m = row0 + lane + 32 * c;
                m = m < p.P ? m : p.P - 1;
                v[c] = load_sf4(p.a_sf + m * p.a_sf_stride, 4 * kb, p.a_chunks, a_aligned);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int n = lane + 32 * c;  // row of the B tile
                const uint8_t* base;
                int row;
                if (MODE == 0) {
                    base = n < 64 ? p.b_sf0 : p.b_sf1;
                    row = w.nt * 64 + (n & 63);
                } else {
                    base = p.b_sf0;
                    row = w.nt * 128 + n;
                }
                v[4 + c] = row < p.b_rows
                               ? load_sf4(base + (static_cast<int64_t>(w.e) * p.b_rows + row) * p.b_sf_stride, 4 * kb,
                                          p.b_chunks, b_aligned)
                               : 0x7F7F7F7Fu;  // padding rows: zero weights, unit scales
            }
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars + 8 * (MB_SFE + ss), ((it / SF_SLOTS) & 1) ^ 1, abort,
                                                            MX_WAIT_NS)))
                return;
            tc_fence_after();
            tmem_st32x8(lane_base + SF_COL + ss * 8, v);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + 8 * (MB_SFF + ss));
        }
    }
}

// MMA issuer (one lane): per item, wait until the accumulator buffer of the
// item's parity is drained; per K block, wait for the operand stage and the
// scale slot, issue four N = 128, K = 32 block-scaled MMAs (chunk j reads
// byte j of the scale columns), and commit so that the stage and the slot are
// released when those MMAs are done; after the item's last K block, commit
// the accumulator to the epilogue.
__device__ __forceinline__ void mx_mma(const MxParams& p, const int* seg, const int* ipre, int total, uint32_t sbase,
                                       uint32_t bars, uint32_t tmem, volatile int* abort)
{
    int it = 0, nitem = 0, last_item = -1;
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
                const uint32_t d = tmem + b * 128;
                const uint32_t sfa = tmem + SF_COL + ss * 8;
                const uint32_t sfb = sfa + 4;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_mx(d, sw128_kmajor_desc(a_addr + j * 32), sw128_kmajor_desc(b_addr + j * 32),
                           idesc_mx(128, 128, static_cast<uint32_t>(j)), sfa | (static_cast<uint32_t>(j) << 30),
                           sfb | (static_cast<uint32_t>(j) << 30), (kb > 0 || j > 0) ? 1u : 0u);
                mma_commit(bars + 8 * (MB_EMPTY + s));
                mma_commit(bars + 8 * (MB_SFE + ss));
            }
        }
        mma_commit(bars + 8 * (MB_AF + b));
        last_item = nitem;
    }
    return;
drain:
    // wait for the MMAs already issued before TMEM is released
    if (last_item >= 0 || it > 0) {
        volatile int no_abort = 0;
        // every MMA issued so far is tracked by the last slot commit
        const int j = it - 1;
        if (j >= 0) mbar_wait_bounded(bars + 8 * (MB_SFE + j % SF_SLOTS), (j / SF_SLOTS) & 1, &no_abort, MX_WAIT_NS / 4);
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
//   gate/up: columns [0,64) hold g, [64,128) u of intermediate columns
//            nt*64 .. nt*64+63; h = SiLU(g) * u; each 32-column half is one
//            MX block of the intermediate row: scale byte and 32 codes.
//   down:    y[pair, nt*128 + c] = topk_w[pair] * acc[c] for c < 128.
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
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bars + 8 * (MB_AF + b), (nitem >> 1) & 1, abort, MX_WAIT_NS)))
            return;
        tc_fence_after();
        const uint32_t col = lane_base + b * 128;
        if (MODE == 0) {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t g[32], u[32];
                __syncwarp();  // the loads are warp-collective
                tmem_ld32_issue(col + half * 32, g);
                tmem_ld_wait(g);
                tmem_ld32_issue(col + 64 + half * 32, u);
                tmem_ld_wait(u);
                if (half == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars + 8 * (MB_AE + b));
                }
                const int c0 = w.nt * 64 + half * 32;  // intermediate column of this block
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
                p.h_scales[static_cast<int64_t>(r) * (p.Ip / 32) + c0 / 32] = sc;
            }
        } else {
            int pair = -1;
            float wt = 0.f;
            if (valid) {
                pair = __ldg(p.sorted_pairs + r);
                if (pair < 0 || pair >= p.P) {
                    atomicOr(p.status, kDevBadPair);
                    pair = -1;
                } else {
                    wt = __ldg(p.topk_w + pair);
                }
            }
            float* dst = pair >= 0 ? p.y + static_cast<int64_t>(pair) * p.H + w.nt * 128 : nullptr;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                __syncwarp();
                tmem_ld32_issue(col + c * 32, v);
                tmem_ld_wait(v);
                if (c == 3) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars + 8 * (MB_AE + b));
                }
                if (!dst || w.nt * 128 + c * 32 >= p.H) continue;
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
            mbar_init(bars + 8 * (MB_FULL + s), 2);   // both producers: arrive + tx
            mbar_init(bars + 8 * (MB_EMPTY + s), 1);  // MMA commit
        }
        for (int s = 0; s < SF_SLOTS; ++s) {
            mbar_init(bars + 8 * (MB_SFF + s), 4);    // four stager warps
            mbar_init(bars + 8 * (MB_SFE + s), 1);    // MMA commit
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
        if ((threadIdx.x & 31) == 0) {
            if (warp == 0) mx_producer_b<MODE>(&tmB0, &tmB1, p, seg, ipre, total, sbase, bars, abort);
            else if (warp == 1) mx_mma(p, seg, ipre, total, sbase, bars, tmem, abort);
            else if (warp == 3) mx_producer_a(&tmA, p, seg, ipre, total, sbase, bars, abort);
        }
    } else if (warp < 8) {
        mx_epilogue<MODE>(p, seg, ipre, total, bars, tmem, abort);
    } else {
        mx_stager<MODE>(p, seg, ipre, total, bars, tmem, abort);
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
// and its H/32 scale bytes into expert order.
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
        const uint32_t* ss = reinterpret_cast<const uint32_t*>(act_scales + t * (H / 32));
        uint32_t* sd = reinterpret_cast<uint32_t*>(sa_sorted + r * (H / 32));
        for (int c = lane; c < n4; c += 32) sd[c] = __ldg(ss + c);
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

size_t ffn_mx_workspace_layout(int64_t T, int H, int I, int k, size_t* off_a, size_t* off_sa, size_t* off_h,
                               size_t* off_sh)
{
    const int64_t P = T * k > 0 ? T * k : 1;
    const int64_t Ip = (static_cast<int64_t>(I) + 127) / 128 * 128;
    size_t o = 256;  // status word
    *off_a = o;
    o = align_up(o + static_cast<size_t>(P) * H, 256);
    *off_sa = o;
    o = align_up(o + static_cast<size_t>(P) * (H / 32), 256);
    *off_h = o;
    o = align_up(o + static_cast<size_t>(P) * Ip, 256);
    *off_sh = o;
    o = align_up(o + static_cast<size_t>(P) * (Ip / 32), 256);
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

    // 2. tensor maps: activations and intermediate [rows, K] with 128-row
    // boxes; gate/up weights with 64-row boxes (64 gate + 64 up rows per
    // tile), down weights with 128-row boxes.  The intermediate's map is I
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
        if (!a.down_only && (!make_tmap_u8(&tmA1, a.a_sorted, 2, dA, sA, 128) ||
                             !make_tmap_u8(&tmG, a.w_gate, 3, dW, sW, 64) ||
                             !make_tmap_u8(&tmU, a.w_up, 3, dW, sW, 64)))
            return cudaErrorNotSupported;
        if (!make_tmap_u8(&tmA2, a.h_codes, 2, dH, sH, 128) || !make_tmap_u8(&tmD, a.w_down, 3, dD, sD, 128))
            return cudaErrorNotSupported;
    }
    const int grid = di.sm_count;

    // 3. gate/up GEMM with the SiLU*up + MX requantisation epilogue
    MxParams g{};
    g.E = E;
    g.num_kb = (H + MX_BK - 1) / MX_BK;
    g.n_tiles = (I + 63) / 64;
    g.P = P;
    g.offsets = a.expert_offsets;
    g.a_sf = a.sa_sorted;
    g.a_sf_stride = H / 32;
    g.a_chunks = H / 32;
    g.b_sf0 = a.s_gate;
    g.b_sf1 = a.s_up;
    g.b_rows = I;
    g.b_sf_stride = H / 32;
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
    d.n_tiles = (H + 127) / 128;
    d.a_sf = a.h_scales;
    d.a_sf_stride = Ip / 32;
    d.a_chunks = I / 32;
    d.b_sf0 = a.s_down;
    d.b_sf1 = a.s_down;
    d.b_rows = H;
    d.b_sf_stride = I / 32;
    d.b_chunks = I / 32;
    if ((err = mx_stage_mark(a, 2, s)) != cudaSuccess) return err;
    if ((err = run_mx<1>(tmA2, tmD, tmD, d, grid, s)) != cudaSuccess) return err;
    return mx_stage_mark(a, 3, s);
}

}  // namespace fp8moe
