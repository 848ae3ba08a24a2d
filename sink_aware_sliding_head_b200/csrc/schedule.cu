// schedule.cu - on-device work list for the persistent attention kernels.
//
// THD packing (attention utils page, nemo_automodel.components.attention.utils:
// cu_seqlens int32 [documents + 1]) and the causal, window-limited document
// mask decide which tiles hold work. One launch of a single 1024-thread block:
//   1. enumerates work items per document: query-major items (a span of query
//      tokens of one KV group) or key-major items (128 keys of one KV group);
//   2. prices each item by the number of tiles it will visit (key tiles for
//      query-major items, 128-row query tiles for key-major ones) - tiles
//      wholly outside the window or another document are never listed;
//   3. counting-sorts the items by price, heaviest first, so that persistent
//      CTAs that take items in list order through a global counter schedule
//      them greedily longest-first (LPT) and finish together.
// Item = int4 {first token, document start, document end, KV head}.
// With padding (valid != nullptr), document d ends after its valid[d] real
// tokens: the trailing padding gets no item, so no kernel visits it as a query
// or a key. The backward's two lists are built by the two blocks of one launch.
#include "common.cuh"

namespace flint {

namespace {

constexpr int kThreads = 1024;
constexpr int kBuckets = 4096;

__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
    int t = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_sums[lane] = t - s;          // exclusive prefix of warp sums
    if (lane == 31) *total = t;
  }
  __syncthreads();
  int r = warp_sums[warp] + x - v;
  __syncthreads();
  return r;
}

__device__ __forceinline__ int item_cost(int mode, int start, int d0, int d1, int span, int W,
                                         int R) {
  if (mode == kModeQuery) {
    int kend = min(start + span, d1);
    int kbeg = W > 0 ? max(d0, start - W + 1) : d0;
    return (kend - kbeg + kTileKeys - 1) / kTileKeys;
  }
  int qend = W > 0 ? min(d1, start + kTileKeys - 1 + W) : d1;
  return (qend - start + R - 1) / R;
}

// One list, built by the whole (1024-thread) block.
__device__ void build_list(const int32_t* __restrict__ cu, const int32_t* __restrict__ valid,
                           int N, int mode, int span, int W, int R, int Hk,
                           int4* __restrict__ items, int* __restrict__ count,
                           int4* __restrict__ tmp_items, int* __restrict__ tmp_cost,
                           int max_items) {
  __shared__ int warp_sums[32];
  __shared__ int total_s;
  __shared__ int chunk_off[kThreads + 1];
  __shared__ int hist[kBuckets];
  for (int b = threadIdx.x; b < kBuckets; b += kThreads) hist[b] = 0;
  __syncthreads();

  // 1+2. enumerate and price, chunk by chunk of documents
  int base = 0;
  for (int dc = 0; dc < N; dc += kThreads) {
    const int d = dc + threadIdx.x;
    int n = 0, d0 = 0, d1 = 0;
    if (d < N) {
      d0 = __ldg(cu + d);
      d1 = __ldg(cu + d + 1);
      if (valid) d1 = d0 + max(0, min(__ldg(valid + d), d1 - d0));
      n = (d1 > d0 ? (d1 - d0 + span - 1) / span : 0) * Hk;
    }
    int ex = block_exclusive_scan(n, warp_sums, &total_s);
    chunk_off[threadIdx.x] = ex;
    if (threadIdx.x == kThreads - 1) chunk_off[kThreads] = ex + n;
    __syncthreads();
    const int ctotal = chunk_off[kThreads];
    for (int f = threadIdx.x; f < ctotal; f += kThreads) {
      int lo = 0, hi = kThreads;                 // last lo with chunk_off[lo] <= f
      while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (chunk_off[mid] <= f) lo = mid; else hi = mid;
      }
      while (chunk_off[lo + 1] <= f) ++lo;       // skip documents with no items
      const int dd = dc + lo;
      const int e0 = __ldg(cu + dd);
      int e1 = __ldg(cu + dd + 1);
      if (valid) e1 = e0 + max(0, min(__ldg(valid + dd), e1 - e0));
      const int local = f - chunk_off[lo];
      const int start = e0 + (local / Hk) * span;
      const int g = local % Hk;
      const int slot = base + f;
      if (slot < max_items) {
        const int c = item_cost(mode, start, e0, e1, span, W, R);
        tmp_items[slot] = make_int4(start, e0, e1, g);
        tmp_cost[slot] = c;
        atomicAdd(&hist[min(c, kBuckets - 1)], 1);
      }
    }
    base += ctotal;
    __syncthreads();
  }
  const int n_items = min(base, max_items);

  // 3. counting sort, heaviest bucket first
  // exclusive scan of hist in descending bucket order -> start cursor per bucket
  const int per = kBuckets / kThreads;           // 4 buckets per thread
  int local[per];
  int sum = 0;
#pragma unroll
  for (int e = 0; e < per; ++e) {
    // thread 0 owns the heaviest buckets
    local[e] = hist[kBuckets - 1 - (threadIdx.x * per + e)];
    sum += local[e];
  }
  int ex = block_exclusive_scan(sum, warp_sums, &total_s);
  __syncthreads();
#pragma unroll
  for (int e = 0; e < per; ++e) {
    hist[kBuckets - 1 - (threadIdx.x * per + e)] = ex;
    ex += local[e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_items; i += kThreads) {
    const int c = min(tmp_cost[i], kBuckets - 1);
    const int pos = atomicAdd(&hist[c], 1);
    items[pos] = tmp_items[i];
  }
  if (threadIdx.x == 0) *count = n_items;
}

struct ListSpec {
  int mode, span;
  int4* items;
  int* count;
  int4* tmp_items;
  int* tmp_cost;
  int max_items;
};

// Block b builds list b (gridDim.x lists, at most 2), independently.
__global__ void __launch_bounds__(kThreads)
build_worklist_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ valid, int N,
                      int W, int R, int Hk, ListSpec l0, ListSpec l1) {
  const ListSpec& L = blockIdx.x == 0 ? l0 : l1;
  build_list(cu, valid, N, L.mode, L.span, W, R, Hk, L.items, L.count, L.tmp_items, L.tmp_cost,
             L.max_items);
}

ListSpec spec(int mode, int span, int4* items, int* count, void* tmp, int max_items) {
  ListSpec l;
  l.mode = mode; l.span = span; l.items = items; l.count = count;
  l.tmp_items = reinterpret_cast<int4*>(tmp);
  l.tmp_cost = reinterpret_cast<int*>(l.tmp_items + max_items);
  l.max_items = max_items;
  return l;
}

}  // namespace

cudaError_t launch_build_worklist(const int32_t* cu, const int32_t* valid, const Resolved& p,
                                  int mode, int span, int4* items, int* count, void* tmp,
                                  int max_items, cudaStream_t st) {
  const ListSpec l = spec(mode, span, items, count, tmp, max_items);
  ProfScope prof(kKWorklist, st);
  build_worklist_kernel<<<1, kThreads, 0, st>>>(cu, valid, p.N, p.W, p.R, p.Hk, l, l);
  return cudaGetLastError();
}

cudaError_t launch_build_worklists2(const int32_t* cu, const int32_t* valid, const Resolved& p,
                                    int mode0, int span0, int4* items0, int* count0, void* tmp0,
                                    int max0, int mode1, int span1, int4* items1, int* count1,
                                    void* tmp1, int max1, cudaStream_t st) {
  const ListSpec l0 = spec(mode0, span0, items0, count0, tmp0, max0);
  const ListSpec l1 = spec(mode1, span1, items1, count1, tmp1, max1);
  ProfScope prof(kKWorklist, st);
  build_worklist_kernel<<<2, kThreads, 0, st>>>(cu, valid, p.N, p.W, p.R, p.Hk, l0, l1);
  return cudaGetLastError();
}

}  // namespace flint
