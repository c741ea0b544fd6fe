// route.cu -- top-k routing with softmax-normalised weights and the stable
// permutation of (token, slot) pairs by expert.
//
// Pages: top-k routes with normalised routing weights ("Exact AVX2 FP8
// arithmetic conversion avoids costly LUT gathers", "Real-checkpoint
// measurements"); a fused router chain gate -> top-k -> dispatch ("Integration
// for GLM-4.6-FP8 and performance tune on H20", gap table row 7); a plan
// step that groups pairs for the grouped gate/up call and whose member
// order is a deterministic rank ("GLM-5.3-Flash EXL3 on CUDA: a whole prompt
// pass routes its experts in one call", "Exactness").
//
// Three launches, no host synchronisation, no atomics on the ordering path:
//   1. route_topk: one warp per token (4 tokens per warp, 32 warps per
//      block).  Logits of a token sit in registers (ceil(E/32) per lane);
//      k rounds of a warp arg-max (value desc, id asc; NaN and -Inf are
//      never selected).  Slot weights: expf(l_j - l_0) / sum (FP32).  The
//      same kernel ranks each pair among the block's earlier pairs of the
//      same expert (per-warp counters in shared memory, tokens in order), and
//      writes the block's per-expert counts.
//   2. route_scan: one block; per expert, exclusive prefix of the block
//      counts in block order, then an exclusive scan over experts.
//   3. route_scatter: pair p goes to offsets[e] + base[block(p)][e] +
//      rank_in_block(p); positions past offsets[E] get -1.
// Every integer output is a pure function of the ids, so it is the same for
// any launch shape and from run to run.
#include <cfloat>
#include <climits>
#include <cstdio>
#include <mutex>

#include "../../include/fp8moe.h"
#include "internal.h"

namespace fp8moe {
namespace {

constexpr int kWarps = 32;
constexpr int kTokPerWarp = kRouteTokensPerBlock / kWarps;  // 4

template <int VPL>
__global__ void __launch_bounds__(kWarps * 32) route_topk_kernel(const float* __restrict__ logits, int64_t T, int E,
                                                                 int k, int32_t* __restrict__ ids,
                                                                 float* __restrict__ w,
                                                                 int32_t* __restrict__ block_hist,
                                                                 int32_t* __restrict__ local_rank)
{
    extern __shared__ int32_t sm[];
    int32_t* warp_cnt = sm;                                     // [kWarps][E]
    int32_t* s_rank = sm + kWarps * E;                          // [128][k]
    int32_t* s_id = s_rank + kRouteTokensPerBlock * k;          // [128][k]
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) warp_cnt[i] = 0;
    for (int i = threadIdx.x; i < kRouteTokensPerBlock * k; i += blockDim.x) s_id[i] = -1;
    __syncthreads();

    const int64_t blk_tok0 = static_cast<int64_t>(blockIdx.x) * kRouteTokensPerBlock;
    for (int tt = 0; tt < kTokPerWarp; ++tt) {
        const int tl = warp * kTokPerWarp + tt;  // token index within the block
        const int64_t t = blk_tok0 + tl;
        if (t >= T) break;
        const float* row = logits + t * E;
        float v[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = lane + 32 * i;
            v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
        }
        uint32_t taken = 0;
        int my_id = -1;
        float my_val = 0.0f, top = 0.0f;
        int nsel = 0;
        for (int j = 0; j < k; ++j) {
            float bv = -INFINITY;
            int be = INT_MAX;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int e = lane + 32 * i;
                const bool sel = (e < E) && !((taken >> i) & 1u) && !isnan(v[i]) && v[i] != -INFINITY;
                if (sel && (be == INT_MAX || v[i] > bv)) {  // ascending e: strict '>' keeps the lower id
                    bv = v[i];
                    be = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
                const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
                if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
                    bv = ov;
                    be = oe;
                }
            }
            if (be == INT_MAX) break;  // nothing selectable is left
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            if (lane == j) {
                my_id = be;
                my_val = bv;
            }
            if (j == 0) top = bv;
            ++nsel;
        }
        const float ex = (lane < nsel) ? expf(my_val - top) : 0.0f;
        float sum = ex;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
        if (lane < k) {
            ids[t * k + lane] = (lane < nsel) ? my_id : -1;
            w[t * k + lane] = (lane < nsel) ? __fdiv_rn(ex, sum) : 0.0f;
        }
        // stable rank among this warp's earlier pairs of the same expert; a
        // token's selected experts are distinct, so lanes never collide
        if (lane < nsel) {
            const int c = warp_cnt[warp * E + my_id];
            s_rank[tl * k + lane] = c;
            s_id[tl * k + lane] = my_id;
            warp_cnt[warp * E + my_id] = c + 1;
        }
        __syncwarp();
    }
    __syncthreads();
    // per expert: exclusive prefix over warps (warp order = token order)
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int ww = 0; ww < kWarps; ++ww) {
            const int c = warp_cnt[ww * E + e];
            warp_cnt[ww * E + e] = run;
            run += c;
        }
        block_hist[static_cast<int64_t>(blockIdx.x) * E + e] = run;
    }
    __syncthreads();
    for (int q = threadIdx.x; q < kRouteTokensPerBlock * k; q += blockDim.x) {
        const int id = s_id[q];
        if (id < 0) continue;
        const int tl = q / k;
        local_rank[blk_tok0 * k + q] = warp_cnt[(tl / kTokPerWarp) * E + id] + s_rank[q];
    }
}

__global__ void __launch_bounds__(1024) route_scan_kernel(int32_t* __restrict__ block_hist, int nblocks, int E,
                                                          int32_t* __restrict__ offsets)
{
    __shared__ int32_t wsum[32];
    const int e = threadIdx.x;
    const int lane = e & 31, warp = e >> 5;
    int run = 0;
    if (e < E) {
        // batches of independent loads, then their running prefix
        for (int b0 = 0; b0 < nblocks; b0 += 16) {
            int c[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                c[j] = (b0 + j < nblocks) ? block_hist[static_cast<int64_t>(b0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (b0 + j < nblocks) block_hist[static_cast<int64_t>(b0 + j) * E + e] = run;
                run += c[j];
            }
        }
    }
    int incl = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = wsum[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, v, off);
            if (lane >= off) v += y;
        }
        wsum[lane] = v;
    }
    __syncthreads();
    const int excl = (warp ? wsum[warp - 1] : 0) + incl - run;
    if (e < E) offsets[e] = excl;
    if (e == E - 1) offsets[E] = excl + run;
}

__global__ void route_scatter_kernel(const int32_t* __restrict__ ids, int64_t P, int k, int E,
                                     const int32_t* __restrict__ block_hist, const int32_t* __restrict__ local_rank,
                                     const int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_pairs)
{
    const int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (p >= P) return;
    const int total = offsets[E];
    const int e = ids[p];
    if (e >= 0) {
        const int64_t b = (p / k) / kRouteTokensPerBlock;
        const int64_t pos = static_cast<int64_t>(offsets[e]) + block_hist[b * E + e] + local_rank[p];
        sorted_pairs[pos] = static_cast<int32_t>(p);
    }
    if (p >= total) sorted_pairs[p] = -1;
}

__global__ void zero_offsets_kernel(int32_t* offsets, int n)
{
    for (int i = threadIdx.x; i < n; i += blockDim.x) offsets[i] = 0;
}

template <int VPL>
size_t topk_smem(int E, int k)
{
    return (static_cast<size_t>(kWarps) * E + 2ull * kRouteTokensPerBlock * k) * sizeof(int32_t);
}

template <int VPL>
cudaError_t run_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* w, int32_t* hist,
                     int32_t* lrank, int nblocks, cudaStream_t s)
{
    const size_t smem = topk_smem<VPL>(E, k);
    if (smem > 48 * 1024) {
        cudaError_t err =
            cudaFuncSetAttribute(route_topk_kernel<VPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    route_topk_kernel<VPL><<<nblocks, kWarps * 32, smem, s>>>(logits, T, E, k, ids, w, hist, lrank);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int32_t* ids, float* w, int32_t* offsets,
                         int32_t* sorted_pairs, int32_t* block_hist, int32_t* local_rank, cudaStream_t s)
{
    if (T == 0 || k == 0) {
        zero_offsets_kernel<<<1, 256, 0, s>>>(offsets, E + 1);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess || T == 0) return err;
        // top_k == 0: nothing is routed; ids/w/sorted_pairs are empty
        return cudaSuccess;
    }
    const int nblocks = static_cast<int>(ceil_div64(T, kRouteTokensPerBlock));
    cudaError_t err;
    if (E <= 64) err = run_topk<2>(logits, T, E, k, ids, w, block_hist, local_rank, nblocks, s);
    else if (E <= 256) err = run_topk<8>(logits, T, E, k, ids, w, block_hist, local_rank, nblocks, s);
    else err = run_topk<32>(logits, T, E, k, ids, w, block_hist, local_rank, nblocks, s);
    if (err != cudaSuccess) return err;
    route_scan_kernel<<<1, 1024, 0, s>>>(block_hist, nblocks, E, offsets);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int64_t P = T * k;
    route_scatter_kernel<<<static_cast<int>(ceil_div64(P, 256)), 256, 0, s>>>(ids, P, k, E, block_hist, local_rank,
                                                                             offsets, sorted_pairs);
    return cudaGetLastError();
}

}  // namespace fp8moe

// ---------------------------------------------------------------------------
// moe_route_noalloc: moe_route for callers that cannot allocate device
// memory at all -- not even the small workspace moe_route asks for.  Typical
// cases: code running inside another runtime's execution hook (an inference
// engine plugin, a custom op inside a framework that owns and pre-plans every
// device byte), or latency-critical paths where the implicit device
// synchronisation of cudaMalloc/cudaFree is not acceptable.  The scratch the
// router needs lives in one file-scope device array instead, which every GPU
// that loads this library holds until the process exits.
namespace {

// Route scratch for one call: block histograms ceil(T/128) x E int32, then
// per-pair block ranks T*top_k int32 (each region 256-byte aligned).  1 MiB
// + 4 KiB covers, for example, T = 16384 tokens with E = 1024 experts and
// top_k = 8.
constexpr size_t kNoAllocScratchBytes = (size_t(1) << 20) + 4096;
__device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

// Device address of g_route_scratch, looked up once per device with that
// device current (in host code the symbol is only a host-side stand-in and
// must not be passed to a kernel).
void* scratch_address(int dev, cudaError_t* err)
{
    static void* addr[64] = {};
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    *err = cudaSuccess;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    if (!addr[dev]) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_route_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

thread_local char g_noalloc_error[160] = "";

}  // namespace

extern "C" const char* moe_route_noalloc_error(void) { return g_noalloc_error; }

extern "C" int moe_route_noalloc(const float* logits, int64_t T, int E, int top_k, int32_t* topk_ids,
                                 float* topk_w, int32_t* expert_offsets, int32_t* sorted_pairs, void* stream)
{
    using namespace fp8moe;
    g_noalloc_error[0] = 0;
    if (T < 0 || E < 1 || E > MOE_MAX_EXPERTS || top_k < 0 || top_k > E || top_k > MOE_MAX_TOP_K)
        return MOE_ERR_INVALID_ARG;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && top_k > 0 && (!logits || !topk_ids || !topk_w || !sorted_pairs)) return MOE_ERR_INVALID_ARG;
    auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!al(logits) || !al(topk_ids) || !al(topk_w) || !al(expert_offsets) || !al(sorted_pairs))
        return MOE_ERR_ALIGNMENT;
    // the same scratch layout moe_route uses inside its workspace
    const int64_t nblocks = ceil_div64(T > 0 ? T : 1, kRouteTokensPerBlock);
    const size_t off_hist = 256;
    const size_t off_rank = align_up(off_hist + static_cast<size_t>(nblocks) * E * 4, 256);
    const size_t need = align_up(off_rank + static_cast<size_t>(T > 0 ? T : 1) * (top_k > 0 ? top_k : 1) * 4, 256);
    if (need > kNoAllocScratchBytes) {
        std::snprintf(g_noalloc_error, sizeof(g_noalloc_error),
                      "route scratch for T=%lld E=%d top_k=%d is %zu bytes; the static array holds %zu",
                      static_cast<long long>(T), E, top_k, need, kNoAllocScratchBytes);
        return MOE_ERR_WORKSPACE;
    }
    DeviceInfo di;
    if (!device_info(&di)) return MOE_ERR_CUDA;
    if (di.major != 10 || di.minor != 0) return MOE_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    cudaError_t err;
    uint8_t* base = static_cast<uint8_t*>(scratch_address(dev, &err));
    if (!base) {
        std::snprintf(g_noalloc_error, sizeof(g_noalloc_error), "cudaGetSymbolAddress: %s", cudaGetErrorString(err));
        return MOE_ERR_CUDA;
    }
    // Nothing in the array has to start at zero: every call writes the
    // histograms and ranks it later reads.
    err = launch_route(logits, T, E, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs,
                       reinterpret_cast<int32_t*>(base + off_hist), reinterpret_cast<int32_t*>(base + off_rank),
                       static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) {
        std::snprintf(g_noalloc_error, sizeof(g_noalloc_error), "launch: %s", cudaGetErrorString(err));
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
