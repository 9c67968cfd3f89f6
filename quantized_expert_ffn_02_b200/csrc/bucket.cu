// bucket.cu -- K3: token -> expert bucketing for batch-union dispatch.
//
// Batch-union (colibri README, "What's implemented": each unique expert of the batch is read
// once and applied to every position that routes to it) needs, per expert, the list of
// (token, rank) entries routed to it.  The iliria page ("What's implemented": grouped CPU MoE,
// a ragged descriptor over the expert slabs) keeps the same kind of ragged table.  Here:
//   cnt[e]      entries routed to expert e
//   off[e]      exclusive prefix sum of cnt (off[E] = the routed entries: T * k, fewer when
//               adaptive top-p dropped some; a dropped entry has slot_of = -1)
//   perm[p]     entry id t * k + rank for routed slot p; slots of one expert are contiguous
//               and in ascending token order (a stable scatter)
//   slot_of[i]  inverse of perm
//   ulist[u]    the experts with cnt > 0, ascending; n_unique of them
// One block of 1024 threads: each of the 32 warps owns a contiguous run of tokens, counts
// its entries per expert, a scan over (warp, expert) gives each warp its base per expert,
// and a second pass places the entries in token order.
#include "internal.cuh"

namespace qe {
namespace {

constexpr int kBucketWarps = 32;

__global__ void __launch_bounds__(kBucketWarps * kWarp)
bucket_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int32_t* __restrict__ cnt,
              int32_t* __restrict__ off, int32_t* __restrict__ perm, int32_t* __restrict__ slot_of,
              int32_t* __restrict__ ulist, int32_t* __restrict__ n_unique) {
    extern __shared__ int32_t sm[];
    int32_t* hist = sm;                              // [kBucketWarps][E]
    int32_t* scan = sm + kBucketWarps * E;           // [E + 1]
    const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
    const int per = (T + kBucketWarps - 1) / kBucketWarps;
    const int t_begin = min(T, warp * per), t_end = min(T, t_begin + per);

    for (int i = threadIdx.x; i < kBucketWarps * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    // 1. per-warp histograms (the k experts of one token are distinct)
    for (int t = t_begin; t < t_end; ++t) {
        if (lane < k) {
            const int e = idx[(size_t)t * k + lane];
            if (e >= 0) hist[warp * E + e] += 1;          // -1: dropped by adaptive top-p
        }
        __syncwarp();
    }
    __syncthreads();
    // 2. exclusive scan over warps, per expert; totals -> scan[e]
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kBucketWarps; ++w) {
            const int c = hist[w * E + e];
            hist[w * E + e] = run;
            run += c;
        }
        scan[e] = run;
        cnt[e] = run;
    }
    __syncthreads();
    // 3. exclusive scan over experts (E <= 1024: one element per thread, Hillis-Steele)
    int v = threadIdx.x < E ? scan[threadIdx.x] : 0;
    int flag = v > 0 ? 1 : 0;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        int add = 0;
        if (threadIdx.x < E && threadIdx.x >= o) add = scan[threadIdx.x - o];
        __syncthreads();
        if (threadIdx.x < E && threadIdx.x >= o) scan[threadIdx.x] += add;
        __syncthreads();
    }
    // scan[] is now inclusive; exclusive = inclusive - own
    if (threadIdx.x < E) off[threadIdx.x] = scan[threadIdx.x] - v;
    if (threadIdx.x == E - 1) off[E] = scan[E - 1];     // the routed slots (fewer than T k after top-p)
    // unique list: the same scan over the flags (cnt > 0)
    __syncthreads();
    const int excl = threadIdx.x < E ? scan[threadIdx.x] - v : 0;
    __syncthreads();
    if (threadIdx.x < E) scan[threadIdx.x] = flag;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        int add = 0;
        if (threadIdx.x < E && threadIdx.x >= o) add = scan[threadIdx.x - o];
        __syncthreads();
        if (threadIdx.x < E && threadIdx.x >= o) scan[threadIdx.x] += add;
        __syncthreads();
    }
    if (threadIdx.x < E && flag) ulist[scan[threadIdx.x] - 1] = threadIdx.x;
    if (threadIdx.x == E - 1) *n_unique = scan[E - 1];
    __syncthreads();
    if (threadIdx.x < E) scan[threadIdx.x] = excl;     // expert base offsets
    __syncthreads();
    // 4. stable scatter: warp w walks its tokens in order
    for (int t = t_begin; t < t_end; ++t) {
        if (lane < k) {
            const int e = idx[(size_t)t * k + lane];
            int p = -1;
            if (e >= 0) {
                p = scan[e] + hist[warp * E + e];
                hist[warp * E + e] += 1;
                perm[p] = t * k + lane;
            }
            slot_of[(size_t)t * k + lane] = p;
        }
        __syncwarp();
    }
}

}  // namespace

static size_t bucket_smem(const LayerDims& L) { return sizeof(int32_t) * ((size_t)kBucketWarps * L.E + L.E + 1); }

cudaError_t prepare_bucket(const LayerDims& L) {
    if (L.E > 1024 || bucket_smem(L) > 227 * 1024) return cudaErrorInvalidValue;
    return cudaFuncSetAttribute(bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

cudaError_t launch_bucket(const LayerDims& L, int T, const Workspace& ws, const Launch& ctx) {
    if (T == 0) return cudaSuccess;
    QE_LAUNCH(ctx, MOE_KERNEL_BUCKET,
              (bucket_kernel<<<1, kBucketWarps * kWarp, bucket_smem(L), ctx.s>>>(
                  ws.idx, T, L.k, L.E, ws.cnt, ws.off, ws.perm, ws.slot_of, ws.ulist, ws.n_unique)));
    return cudaSuccess;
}

}  // namespace qe
