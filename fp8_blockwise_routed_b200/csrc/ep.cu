// ep.cu -- expert parallelism across `world` GPUs: the pieces of the layer
// that change when each GPU owns E/world experts and each token has a home
// GPU.  The exchange itself (rows between GPUs) is the caller's collective.
//
// Reading of the pages: the layer shards by expert with one exchange step
// per side; to keep a row's bits independent of the sharding, the k slot
// rows of a token are brought to its home GPU and summed there in slot order
// (no floating-point all-reduce).  "GLM-5.3-Flash EXL3 on CUDA ...", the
// exactness note (member order a deterministic rank; a row's bits do not
// depend on how many rows share a call) is the property kept here.
//
// Every rank runs the router over all T tokens, so the ids are the same
// everywhere and both sides of the exchange follow from them:
//   owner(p) = id(p) / (E/world), home(p) = token(p) / T_home.
// Pairs are counting-sorted twice, by (owner, home) and by (home, owner),
// with the stable permutation of the routing step (pair order inside each
// key).  Rank r sends, to each home h, its pairs of key (r, h) in pair order;
// home h receives from each owner o the pairs of key (h, o) in pair order:
// the same rows in the same order, so no indices travel with the rows.
//   send_rows[p]  = position of p among rank r's outgoing rows (-1: p is not
//                   rank r's), the y row the down GEMM writes p to;
//   recv_rows[t', j] = position of home token t' slot j among the incoming
//                   rows (-1: empty slot), read by moe_combine_rows.
#include "../../include/fp8moe.h"
#include "internal.h"

namespace fp8moe {
namespace {

__global__ void ep_keys_kernel(const int32_t* __restrict__ ids, int64_t P, int k, int E, int world, int rank,
                               int64_t T_home, int32_t* __restrict__ local_ids, int32_t* __restrict__ key_oh,
                               int32_t* __restrict__ key_ho)
{
    const int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (p >= P) return;
    const int id = ids[p];
    const int per = E / world;
    if (id < 0 || id >= E) {
        local_ids[p] = -1;
        key_oh[p] = -1;
        key_ho[p] = -1;
        return;
    }
    const int o = id / per;
    const int h = static_cast<int>((p / k) / T_home);
    local_ids[p] = (o == rank) ? id - o * per : -1;
    key_oh[p] = o * world + h;
    key_ho[p] = h * world + o;
}

__global__ void ep_rows_kernel(const int32_t* __restrict__ sorted_oh, const int32_t* __restrict__ offs_oh,
                               const int32_t* __restrict__ sorted_ho, const int32_t* __restrict__ offs_ho, int world,
                               int rank, int k, int64_t T_home, int32_t* __restrict__ send_rows,
                               int32_t* __restrict__ recv_rows)
{
    const int s0 = offs_oh[rank * world], s1 = offs_oh[rank * world + world];
    const int r0 = offs_ho[rank * world], r1 = offs_ho[rank * world + world];
    const int n = (s1 - s0) > (r1 - r0) ? (s1 - s0) : (r1 - r0);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        if (s0 + i < s1) send_rows[sorted_oh[s0 + i]] = i;
        if (r0 + i < r1) {
            const int64_t p = sorted_ho[r0 + i];
            const int64_t t_local = p / k - static_cast<int64_t>(rank) * T_home;
            recv_rows[t_local * k + (p % k)] = i;
        }
    }
}

size_t ep_layout(int64_t T, int k, int world, size_t* off_koh, size_t* off_kho, size_t* off_soh, size_t* off_sho,
                 size_t* off_perm)
{
    const size_t P = static_cast<size_t>(T > 0 ? T : 1) * (k > 0 ? k : 1);
    size_t o = 256;  // status word
    *off_koh = o;
    o = align_up(o + P * 4, 256);
    *off_kho = o;
    o = align_up(o + P * 4, 256);
    *off_soh = o;
    o = align_up(o + P * 4, 256);
    *off_sho = o;
    o = align_up(o + P * 4, 256);
    *off_perm = o;
    return o + moe_route_workspace_bytes(T, world * world, k);
}

}  // namespace
}  // namespace fp8moe

using namespace fp8moe;

namespace {

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int dev_ok()
{
    DeviceInfo di;
    if (!device_info(&di)) return MOE_ERR_CUDA;
    return (di.major == 10 && di.minor == 0) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

size_t moe_ep_plan_workspace_bytes(int64_t T, int top_k, int world)
{
    if (T < 0 || top_k < 1 || world < 1 || world * world > MOE_MAX_EXPERTS) return 0;
    size_t a, b, c, d, e;
    return ep_layout(T, top_k, world, &a, &b, &c, &d, &e);
}

int moe_ep_plan(const int32_t* topk_ids, int64_t T, int top_k, int E, int world, int rank, int64_t T_home,
                int32_t* local_ids, int32_t* send_rows, int32_t* recv_rows, int32_t* offs_oh, int32_t* offs_ho,
                void* ws, size_t ws_bytes, void* stream)
{
    if (T < 0 || top_k < 1 || top_k > MOE_MAX_TOP_K || E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_INVALID_ARG;
    if (world < 1 || world * world > MOE_MAX_EXPERTS || rank < 0 || rank >= world || E % world != 0)
        return MOE_ERR_INVALID_ARG;
    if (T_home < 1 || T_home * world < T) return MOE_ERR_INVALID_ARG;
    if (T > (int64_t(1) << 31) / top_k - 1) return MOE_ERR_UNSUPPORTED;
    if (!ws || !offs_oh || !offs_ho || (T > 0 && (!topk_ids || !local_ids || !send_rows || !recv_rows)))
        return MOE_ERR_INVALID_ARG;
    if (!al16(topk_ids) || !al16(local_ids) || !al16(send_rows) || !al16(recv_rows) || !al16(offs_oh) ||
        !al16(offs_ho) || !al16(ws))
        return MOE_ERR_ALIGNMENT;
    size_t off_koh, off_kho, off_soh, off_sho, off_perm;
    if (ws_bytes < ep_layout(T, top_k, world, &off_koh, &off_kho, &off_soh, &off_sho, &off_perm))
        return MOE_ERR_WORKSPACE;
    if (int r = dev_ok()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaError_t err = cudaMemsetAsync(ws, 0, sizeof(int), s);
    const int64_t P = T * top_k;
    const int keys = world * world;
    if (err == cudaSuccess && P > 0) err = cudaMemsetAsync(send_rows, 0xFF, static_cast<size_t>(P) * 4, s);
    if (err == cudaSuccess && T_home * top_k > 0)
        err = cudaMemsetAsync(recv_rows, 0xFF, static_cast<size_t>(T_home) * top_k * 4, s);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    auto* koh = reinterpret_cast<int32_t*>(w + off_koh);
    auto* kho = reinterpret_cast<int32_t*>(w + off_kho);
    auto* soh = reinterpret_cast<int32_t*>(w + off_soh);
    auto* sho = reinterpret_cast<int32_t*>(w + off_sho);
    if (P > 0) {
        ep_keys_kernel<<<static_cast<int>(ceil_div64(P, 256)), 256, 0, s>>>(topk_ids, P, top_k, E, world, rank,
                                                                           T_home, local_ids, koh, kho);
        if ((err = cudaGetLastError()) != cudaSuccess) return MOE_ERR_CUDA;
    }
    // both permutations use the same router scratch, one after the other
    uint8_t* pw = w + off_perm;
    size_t a_arr, a_hist, a_rank;
    route_ws_layout(T, keys, top_k, &a_arr, &a_hist, &a_rank);
    for (int pass = 0; pass < 2; ++pass) {
        err = launch_permute(pass ? kho : koh, T, keys, top_k, pass ? offs_ho : offs_oh, pass ? sho : soh,
                             reinterpret_cast<int32_t*>(pw + a_hist), reinterpret_cast<int32_t*>(pw + a_rank),
                             reinterpret_cast<int*>(pw + a_arr), s);
        if (err != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (P > 0) {
        ep_rows_kernel<<<64, 256, 0, s>>>(soh, offs_oh, sho, offs_ho, world, rank, top_k, T_home, send_rows,
                                          recv_rows);
        if ((err = cudaGetLastError()) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

int moe_permute(const int32_t* ids, int64_t T, int E, int top_k, int32_t* expert_offsets, int32_t* sorted_pairs,
                void* ws, size_t ws_bytes, void* stream)
{
    if (T < 0 || E < 1 || E > MOE_MAX_EXPERTS || top_k < 0 || top_k > MOE_MAX_TOP_K) return MOE_ERR_INVALID_ARG;
    if (T > (int64_t(1) << 31) / (top_k > 0 ? top_k : 1) - 1) return MOE_ERR_UNSUPPORTED;
    if (!expert_offsets || !ws || (T > 0 && top_k > 0 && (!ids || !sorted_pairs))) return MOE_ERR_INVALID_ARG;
    if (!al16(ids) || !al16(expert_offsets) || !al16(sorted_pairs) || !al16(ws)) return MOE_ERR_ALIGNMENT;
    if (ws_bytes < moe_route_workspace_bytes(T, E, top_k)) return MOE_ERR_WORKSPACE;
    if (int r = dev_ok()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(ws);
    if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
    size_t a_arr, a_hist, a_rank;
    route_ws_layout(T, E, top_k, &a_arr, &a_hist, &a_rank);
    const cudaError_t err = launch_permute(ids, T, E, top_k, expert_offsets, sorted_pairs,
                                           reinterpret_cast<int32_t*>(w + a_hist),
                                           reinterpret_cast<int32_t*>(w + a_rank), reinterpret_cast<int*>(w + a_arr),
                                           s);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
