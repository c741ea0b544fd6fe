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
//   1. route_topk: one warp per token, 8 tokens per block, so the whole GPU
//      takes part.  A token's logits sit in registers (ceil(E/32) per
//      lane); k rounds of a warp arg-max (value desc, id asc; NaN and -Inf
//      are never selected).  Slot weights: expf(l_j - l_0) / sum (FP32).
//      The same launch can carry the activation quantiser in its trailing
//      blocks (moe_route_quant), which needs no routing result.
//   2. route_rank: one block per 128 tokens.  A pair's rank among the
//      block's earlier pairs of the same expert comes from a warp match
//      (lanes in order) plus per-warp counts in shared memory (warps in
//      order); the block writes its per-expert counts.  The last block to
//      finish (an arrival counter) scans the counts: per expert, exclusive
//      prefix over blocks in block order, then an exclusive scan over
//      experts -> expert_offsets.
//   3. route_scatter: pair p goes to offsets[e] + base[block(p)][e] +
//      rank_in_block(p); positions past offsets[E] get -1.
// Every integer output is a pure function of the ids, so it is the same for
// any launch shape and from run to run.
#include <cuda.h>

#include <cfloat>
#include <climits>
#include <cstdio>
#include <mutex>

#include "../../include/fp8moe.h"
#include "internal.h"
#include "quant_body.cuh"

namespace fp8moe {
namespace {

constexpr int kTopkWarps = 8;     // tokens per top-k block
constexpr int kRankThreads = 1024;

// Top-k of one token by one warp; writes ids[t*k + j], w[t*k + j].
template <int VPL>
__device__ __forceinline__ void topk_token(const float* __restrict__ row, int E, int k, int32_t* __restrict__ ids,
                                           float* __restrict__ w, int lane)
{
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
        ids[lane] = (lane < nsel) ? my_id : -1;
        w[lane] = (lane < nsel) ? __fdiv_rn(ex, sum) : 0.0f;
    }
}

// Blocks [0, n_topk): one token per warp.  Blocks [n_topk, gridDim.x): the
// activation quantiser (optional).  Block 0 also resets the rank kernel's
// arrival counter (this launch precedes it in stream order).
template <int VPL>
__global__ void __launch_bounds__(kTopkWarps * 32) route_topk_kernel(const float* __restrict__ logits, int64_t T,
                                                                     int E, int k, int shared,
                                                                     int32_t* __restrict__ ids,
                                                                     float* __restrict__ w, int* __restrict__ arrivals,
                                                                     int64_t n_topk, const uint4* __restrict__ qx,
                                                                     int64_t q_groups, uint8_t* __restrict__ q_codes,
                                                                     float* __restrict__ q_scales)
{
    if (blockIdx.x >= n_topk) {
        quant::groups(qx, q_groups, q_codes, q_scales, blockIdx.x - n_topk, gridDim.x - n_topk);
        return;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *arrivals = 0;
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kTopkWarps + (threadIdx.x >> 5);
    if (t >= T) return;
    const int kout = k + shared;  // the shared-expert slot, if any, follows the top-k
    topk_token<VPL>(logits + t * E, E, k, ids + t * kout, w + t * kout, lane);
    if (shared && lane == 0) {
        ids[t * kout + k] = E;
        w[t * kout + k] = 1.0f;
    }
}

// One block per kRouteTokensPerBlock tokens; pairs of the block are taken
// in rounds of kRankThreads (one per thread, in pair order).
__global__ void __launch_bounds__(kRankThreads) route_rank_kernel(const int32_t* __restrict__ ids, int64_t T, int E,
                                                                  int k, int32_t* __restrict__ block_hist,
                                                                  int32_t* __restrict__ local_rank,
                                                                  int* __restrict__ arrivals,
                                                                  int32_t* __restrict__ offsets)
{
    extern __shared__ int32_t sm[];
    int32_t* cnt = sm;                         // [32 warps][E]
    int32_t* base = sm + 32 * E;               // [E] pairs of each expert in earlier rounds
    __shared__ int s_last;
    __shared__ int32_t wsum[32];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokensPerBlock;
    const int64_t ntok = (T - t0) < kRouteTokensPerBlock ? (T - t0) : kRouteTokensPerBlock;
    const int npairs = static_cast<int>(ntok) * k;
    const int64_t p0 = t0 * k;
    for (int i = threadIdx.x; i < E; i += blockDim.x) base[i] = 0;

    for (int r0 = 0; r0 < npairs; r0 += kRankThreads) {
        for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) cnt[i] = 0;
        __syncthreads();
        const int q = r0 + threadIdx.x;
        int id = (q < npairs) ? __ldg(ids + p0 + q) : -1;
        if (id >= E) id = -1;  // cannot come from route_topk; never ranked
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, id);
        const int rank_w = __popc(peers & lt_mask);
        if (id >= 0 && rank_w == 0) cnt[warp * E + id] = __popc(peers);
        __syncthreads();
        // per expert: exclusive prefix over warps (warp order = pair order)
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int run = base[e];
            for (int ww = 0; ww < 32; ++ww) {
                const int c = cnt[ww * E + e];
                cnt[ww * E + e] = run;
                run += c;
            }
            base[e] = run;
        }
        __syncthreads();
        if (id >= 0) local_rank[p0 + q] = cnt[warp * E + id] + rank_w;
        __syncthreads();
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) block_hist[static_cast<int64_t>(blockIdx.x) * E + e] = base[e];

    // Arrival: the last block scans every block's counts.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(arrivals, 1) == static_cast<int>(gridDim.x) - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int nblocks = gridDim.x;
    const int e = threadIdx.x;  // one thread per expert (E <= 1024)
    int run = 0;
    if (e < E) {
        // batches of independent loads, then their running prefix; counts of
        // the other blocks are read from L2 (written before their arrival)
        for (int b0 = 0; b0 < nblocks; b0 += 16) {
            int c[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                c[j] = (b0 + j < nblocks) ? __ldcg(block_hist + static_cast<int64_t>(b0 + j) * E + e) : 0;
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
    if (e >= 0 && e < E) {
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

size_t rank_smem(int E) { return (33ull * E) * sizeof(int32_t); }

}  // namespace

cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int32_t* ids, float* w, int32_t* offsets,
                         int32_t* sorted_pairs, int32_t* block_hist, int32_t* local_rank, int* arrivals,
                         const QuantArgs* quant, cudaStream_t s, int shared)
{
    int64_t q_groups = 0, q_blocks = 0;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    if (quant && quant->T > 0) {
        q_groups = quant->T * (quant->H / 128);
        q_blocks = quant::blocks_for(q_groups, di.sm_count);
    }
    if (T == 0 || k == 0) {
        zero_offsets_kernel<<<1, 256, 0, s>>>(offsets, E + 1);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess || q_blocks == 0) return err;
        // top_k == 0 or T == 0: nothing is routed; ids/w/sorted_pairs are empty
        route_topk_kernel<2><<<static_cast<int>(q_blocks), kTopkWarps * 32, 0, s>>>(
            logits, 0, E, k, 0, ids, w, arrivals, 0, reinterpret_cast<const uint4*>(quant->x), q_groups, quant->codes,
            quant->scales);
        return cudaGetLastError();
    }
    const int64_t n_topk = ceil_div64(T, kTopkWarps);
    const int grid = static_cast<int>(n_topk + q_blocks);
    const uint4* qx = quant ? reinterpret_cast<const uint4*>(quant->x) : nullptr;
    uint8_t* qc = quant ? quant->codes : nullptr;
    float* qs = quant ? quant->scales : nullptr;
    if (E <= 64)
        route_topk_kernel<2><<<grid, kTopkWarps * 32, 0, s>>>(logits, T, E, k, shared, ids, w, arrivals, n_topk, qx,
                                                               q_groups, qc, qs);
    else if (E <= 256)
        route_topk_kernel<8><<<grid, kTopkWarps * 32, 0, s>>>(logits, T, E, k, shared, ids, w, arrivals, n_topk, qx,
                                                               q_groups, qc, qs);
    else
        route_topk_kernel<32><<<grid, kTopkWarps * 32, 0, s>>>(logits, T, E, k, shared, ids, w, arrivals, n_topk, qx,
                                                                q_groups, qc, qs);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int nblocks = static_cast<int>(ceil_div64(T, kRouteTokensPerBlock));
    const size_t smem = rank_smem(E);
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(route_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem));
        if (err != cudaSuccess) return err;
    }
    // the pairs include the shared slot (id E), which the ranking skips
    const int kp = k + shared;
    route_rank_kernel<<<nblocks, kRankThreads, smem, s>>>(ids, T, E, kp, block_hist, local_rank, arrivals, offsets);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int64_t P = T * kp;
    route_scatter_kernel<<<static_cast<int>(ceil_div64(P, 256)), 256, 0, s>>>(ids, P, kp, E, block_hist, local_rank,
                                                                             offsets, sorted_pairs);
    return cudaGetLastError();
}

cudaError_t launch_permute(const int32_t* ids, int64_t T, int E, int k, int32_t* offsets, int32_t* sorted_pairs,
                           int32_t* block_hist, int32_t* local_rank, int* arrivals, cudaStream_t s)
{
    if (T == 0 || k == 0) {
        zero_offsets_kernel<<<1, 256, 0, s>>>(offsets, E + 1);
        return cudaGetLastError();
    }
    // the rank kernel's arrival counter starts at zero (route_topk resets it
    // on the routing path)
    cudaError_t err = cudaMemsetAsync(arrivals, 0, sizeof(int), s);
    if (err != cudaSuccess) return err;
    const int nblocks = static_cast<int>(ceil_div64(T, kRouteTokensPerBlock));
    const size_t smem = rank_smem(E);
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(route_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem));
        if (err != cudaSuccess) return err;
    }
    route_rank_kernel<<<nblocks, kRankThreads, smem, s>>>(ids, T, E, k, block_hist, local_rank, arrivals, offsets);
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

// Identity of the calling thread's current CUDA context (the driver's
// cuCtxGetCurrent and cuCtxGetId, reached through the runtime's entry-point
// query so that libcuda need not be linked).  A device reset, or the release
// and re-creation of the primary context, gives a new id, and with it new
// module addresses.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long* id)
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_route_scratch in the current context.  In host code the
// symbol is only a host-side stand-in and must not be passed to a kernel.
// The address is looked up (cudaGetSymbolAddress) the first time a context
// calls, with its device current, and cached per device together with the
// context's id; a call from a different context (after a device reset, for
// instance) looks it up again, so a stale address is never used.
void* scratch_address(int dev, cudaError_t* err)
{
    static void* addr[64] = {};
    static unsigned long long ctx_of[64] = {};
    static std::mutex mu;
    *err = cudaSuccess;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    unsigned long long ctx = 0;
    const bool known = current_context_id(&ctx);  // false before the runtime made a context current
    if (!known || !addr[dev] || ctx_of[dev] != ctx) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_route_scratch);  // creates the context if there was none
        if (*err != cudaSuccess) return nullptr;
        if (!current_context_id(&ctx)) {
            *err = cudaErrorDeviceUninitialized;
            return nullptr;
        }
        addr[dev] = p;
        ctx_of[dev] = ctx;
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
    // moe_route's cap on T (int32 pair indices), before any size arithmetic
    if (T > (int64_t(1) << 31) / (top_k > 0 ? top_k : 1) - 1) return MOE_ERR_UNSUPPORTED;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && top_k > 0 && (!logits || !topk_ids || !topk_w || !sorted_pairs)) return MOE_ERR_INVALID_ARG;
    auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!al(logits) || !al(topk_ids) || !al(topk_w) || !al(expert_offsets) || !al(sorted_pairs))
        return MOE_ERR_ALIGNMENT;
    // the layout moe_route uses inside its workspace: the arrival counter in
    // the first 256 bytes, then the block histograms and the pair ranks
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
    // counter, histograms and ranks it later reads.
    err = launch_route(logits, T, E, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs,
                       reinterpret_cast<int32_t*>(base + off_hist), reinterpret_cast<int32_t*>(base + off_rank),
                       reinterpret_cast<int*>(base), nullptr, static_cast<cudaStream_t>(stream), 0);
    if (err != cudaSuccess) {
        std::snprintf(g_noalloc_error, sizeof(g_noalloc_error), "launch: %s", cudaGetErrorString(err));
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
