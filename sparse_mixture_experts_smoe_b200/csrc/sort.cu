// sort.cu -- the reordering step (smoe_sort): a stable counting sort of the
// T*k slots by expert id, and the per-expert offsets.
//
// The pages name "reordering operations" fused into ParallelLinear (sourcepulse.org
// summary, "How It Works") and call the expert-sorted layout "grouped" (library
// page of arXiv 2403.08245, review 1 summary).  Three launches (one, sort_small_kernel,
// when the slots fit one chunk and E <= 128):
//   1. count:   each block histograms a chunk of kSortChunk slots (shared-memory
//               atomics; counts are order-free).
//   2. scan:    one block turns the [blocks][E] counts into per-block bases
//               (expert-major, block-minor) and the exclusive offsets.
//   3. scatter: each block walks its chunk in rounds of 256 slots in slot order;
//               within a round, __match_any_sync gives each lane its rank among
//               same-expert lanes of its warp, and per-warp counts are scanned
//               across warps, so equal ids keep ascending slot order (stable).
#include <mutex>

#include "common.cuh"

namespace smoe {
namespace {

constexpr int kSortThreads = 256;
constexpr int kSortChunk = 4096;
constexpr int kSortMaxE = 1024;

__global__ void __launch_bounds__(kSortThreads)
sort_count_kernel(const int32_t* __restrict__ idx, int S, int E, int32_t* __restrict__ counts,
                  unsigned* err) {
  __shared__ int hist[kSortMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kSortChunk;
  const int end = min(S, base + kSortChunk);
  bool bad = false;
  for (int p = base + threadIdx.x; p < end; p += blockDim.x) {
    const int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    else bad = true;
  }
  if (bad) report_error(err, ERRBIT_DATA);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(size_t)blockIdx.x * E + e] = hist[e];
}

// counts[b][e] -> base[b][e] = offsets[e] + sum_{b' < b} counts[b'][e] (in place)
__global__ void __launch_bounds__(kSortThreads)
sort_scan_kernel(int32_t* __restrict__ counts, int n_blocks, int E, int32_t* __restrict__ offsets) {
  __shared__ int tot[kSortMaxE];
  __shared__ int warp_sums[kSortThreads / 32];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int b = 0; b < n_blocks; ++b) s += counts[(size_t)b * E + e];
    tot[e] = s;
  }
  __syncthreads();
  // exclusive scan of tot[0..E) in chunks of blockDim.x
  int carry = 0;
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    const int v = e < E ? tot[e] : 0;
    int incl = v;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int wpre = 0;
    for (int w = 0; w < warp; ++w) wpre += warp_sums[w];
    int chunk_total = 0;
    for (int w = 0; w < kSortThreads / 32; ++w) chunk_total += warp_sums[w];
    const int excl = carry + wpre + incl - v;
    __syncthreads();
    if (e < E) {
      offsets[e] = excl;
      int run = excl;
      for (int b = 0; b < n_blocks; ++b) {
        const int c = counts[(size_t)b * E + e];
        counts[(size_t)b * E + e] = run;
        run += c;
      }
    }
    carry += chunk_total;
  }
  if (threadIdx.x == 0) offsets[E] = carry;
}

// Stable placement of the slots [chunk0, chunk_end) given each expert's running
// position run[e] (shared memory, advanced in place): rounds of kSortThreads slots
// in slot order; __match_any_sync ranks each lane among same-expert lanes of its
// warp, and per-warp counts are scanned across warps, so equal ids keep ascending
// slot order.
__device__ __forceinline__ void scatter_chunk(const int32_t* __restrict__ idx, int E, int chunk0,
                                              int chunk_end, int* run,
                                              int (*wcnt)[kSortMaxE / 4 + 1],
                                              int32_t* __restrict__ sorted_slot,
                                              int32_t* __restrict__ inv) {
  // wcnt holds up to kSortMaxE/4 experts per pass; larger E loops in passes below
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kPass = kSortMaxE / 4;
  for (int r0 = chunk0; r0 < chunk_end; r0 += kSortThreads) {
    const int p = r0 + threadIdx.x;
    int e = p < chunk_end ? idx[p] : -1;
    if (e >= E) e = -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & ((1u << lane) - 1u));
    const bool leader = rank == 0;
    int pos = -1;
    for (int e0 = 0; e0 < E; e0 += kPass) {  // experts [e0, e0 + kPass) per pass
      const int ne = min(kPass, E - e0);
      for (int q = threadIdx.x; q < (kSortThreads / 32) * ne; q += blockDim.x)
        wcnt[q / ne][q % ne] = 0;
      __syncthreads();
      const bool mine = e >= e0 && e < e0 + ne;
      if (mine && leader) wcnt[warp][e - e0] = __popc(same);
      __syncthreads();
      // exclusive scan over warps per expert, starting at the running position
      for (int q = threadIdx.x; q < ne; q += blockDim.x) {
        int acc = run[e0 + q];
        for (int w = 0; w < kSortThreads / 32; ++w) {
          const int c = wcnt[w][q];
          wcnt[w][q] = acc;
          acc += c;
        }
        run[e0 + q] = acc;
      }
      __syncthreads();
      if (mine) pos = wcnt[warp][e - e0] + rank;
      __syncthreads();
    }
    if (e >= 0 && pos >= 0) {
      sorted_slot[pos] = p;
      if (inv) inv[p] = pos;
    }
  }
}

__global__ void __launch_bounds__(kSortThreads)
sort_scatter_kernel(const int32_t* __restrict__ idx, int S, int E,
                    const int32_t* __restrict__ base, int32_t* __restrict__ sorted_slot,
                    int32_t* __restrict__ inv) {
  __shared__ int run[kSortMaxE];                              // running position per expert
  __shared__ int wcnt[kSortThreads / 32][kSortMaxE / 4 + 1];  // per-warp counts, per round
  for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = base[(size_t)blockIdx.x * E + e];
  __syncthreads();
  const int chunk0 = blockIdx.x * kSortChunk;
  scatter_chunk(idx, E, chunk0, min(S, chunk0 + kSortChunk), run, wcnt, sorted_slot, inv);
}

// The three steps in one block, for at most one chunk of slots and kSortSmallE
// experts (a decode-sized batch): one launch instead of three.
constexpr int kSortSmallE = 128;

__global__ void __launch_bounds__(kSortThreads)
sort_small_kernel(const int32_t* __restrict__ idx, int S, int E, int32_t* __restrict__ sorted_slot,
                  int32_t* __restrict__ offsets, int32_t* __restrict__ inv, unsigned* err) {
  __shared__ int run[kSortMaxE];
  __shared__ int wcnt[kSortThreads / 32][kSortMaxE / 4 + 1];
  for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int p = threadIdx.x; p < S; p += blockDim.x) {
    const int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&run[e], 1);
    else bad = true;
  }
  if (bad) report_error(err, ERRBIT_DATA);
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive prefix sum (E <= kSortSmallE)
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      const int c = run[e];
      run[e] = acc;
      offsets[e] = acc;
      acc += c;
    }
    offsets[E] = acc;
  }
  __syncthreads();
  scatter_chunk(idx, E, 0, S, run, wcnt, sorted_slot, inv);
}

}  // namespace

size_t sort_workspace_bytes(int T_, int k, int E) {
  const size_t S = (size_t)T_ * k;
  const size_t nb = (S + kSortChunk - 1) / kSortChunk;
  return nb * (size_t)E * sizeof(int32_t);
}

int sort_launches(int T_, int k, int E) {
  return (T_ * k <= kSortChunk && E <= kSortSmallE) ? 1 : 3;
}

cudaError_t launch_sort(const int32_t* idx, int T_, int k, int E, int32_t* sorted_slot,
                        int32_t* offsets, void* ws, unsigned* err, cudaStream_t s, int32_t* inv) {
  const int S = T_ * k;
  if (sort_launches(T_, k, E) == 1) {
    sort_small_kernel<<<1, kSortThreads, 0, s>>>(idx, S, E, sorted_slot, offsets, inv, err);
    return cudaGetLastError();
  }
  const int nb = cdiv(S, kSortChunk);
  int32_t* counts = (int32_t*)ws;
  sort_count_kernel<<<nb, kSortThreads, 0, s>>>(idx, S, E, counts, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sort_scan_kernel<<<1, kSortThreads, 0, s>>>(counts, nb, E, offsets);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sort_scatter_kernel<<<nb, kSortThreads, 0, s>>>(idx, S, E, counts, sorted_slot, inv);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the sort (smoe_sort_static in smoe.h).
//
// Some callers have no way to obtain device memory for a workspace: code that
// runs inside a memory-planned inference runtime which hands kernels only their
// inputs and outputs, or code called where cudaMalloc must not be used (for
// example while work is being captured into a CUDA graph, where an allocation
// would synchronise or fall outside the graph).  For them the per-block expert
// counts live in this fixed device array instead of a caller workspace.
// Every GPU that loads the library holds the array until the process exits.
// ---------------------------------------------------------------------------
constexpr int kSortStaticCounts = 1 << 16;  // int32 entries: 256 KB per device
static __device__ __align__(256) int32_t g_sort_static_counts[kSortStaticCounts];

namespace {
// Device address of the array for the current device, resolved on the first
// call made with that device current (the host-side symbol is only a stand-in
// and must never be passed to a kernel).
int32_t* sort_static_scratch(cudaError_t* status) {
  static std::mutex mu;
  static int32_t* ptrs[128] = {};
  int dev = 0;
  *status = cudaGetDevice(&dev);
  if (*status != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 128) {
    *status = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    int32_t* p = nullptr;
    *status = cudaGetSymbolAddress((void**)&p, g_sort_static_counts);
    if (*status != cudaSuccess) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}
}  // namespace

}  // namespace smoe

extern "C" int smoe_sort_static(const int32_t* topk_idx, int T, int k, int E,
                                int32_t* sorted_slot, int32_t* expert_offsets, void* stream) {
  using namespace smoe;
  if (T < 0 || k <= 0 || E <= 0 || E > kSortMaxE)
    return api_fail(SMOE_ERR_INVALID_ARG, "bad sizes (E <= %d)", kSortMaxE);
  if ((long long)T * k > 0x7fffffffLL)
    return api_fail(SMOE_ERR_INVALID_ARG, "T*k too large for 32-bit indexing");
  if (!expert_offsets) return api_fail(SMOE_ERR_INVALID_ARG, "expert_offsets is NULL");
  const size_t need = sort_workspace_bytes(T, k, E);
  if (need > sizeof(g_sort_static_counts))
    return api_fail(SMOE_ERR_INVALID_ARG,
                    "smoe_sort_static: %zu bytes of counts needed (ceil(T*k/%d) * E * 4) but the "
                    "static scratch holds %zu; use smoe_sort with a workspace",
                    need, kSortChunk, sizeof(g_sort_static_counts));
  cudaStream_t s = (cudaStream_t)stream;
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(expert_offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s);
    return e == cudaSuccess ? SMOE_OK
                            : api_fail(SMOE_ERR_CUDA, "smoe_sort_static: %s", cudaGetErrorString(e));
  }
  if (!topk_idx || !sorted_slot) return api_fail(SMOE_ERR_INVALID_ARG, "topk_idx/sorted_slot is NULL");
  cudaError_t st;
  int32_t* scratch = sort_static_scratch(&st);
  if (!scratch) return api_fail(SMOE_ERR_CUDA, "smoe_sort_static scratch: %s", cudaGetErrorString(st));
  unsigned* err = api_error_word(&st);
  if (!err) return api_fail(SMOE_ERR_CUDA, "smoe_sort_static error word: %s", cudaGetErrorString(st));
  // the counts are fully rewritten by every call, so nothing needs clearing first
  st = launch_sort(topk_idx, T, k, E, sorted_slot, expert_offsets, scratch, err, s);
  return st == cudaSuccess ? SMOE_OK
                           : api_fail(SMOE_ERR_CUDA, "smoe_sort_static: %s", cudaGetErrorString(st));
}
