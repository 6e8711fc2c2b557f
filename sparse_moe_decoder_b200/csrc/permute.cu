// Dispatch permutation for the grouped experts.
//
// The pages name no dispatch step; it follows from sparse experts (ZONOS2 Technical Report
// digest, "method overview and architecture", item 5: each token visits its top-k of 16
// experts).  Rows are ordered by expert, then by token (stable), so every output is
// bit-exact and deterministic:
//   counts[e], offsets = exclusive prefix of counts, perm[row] = t, inv_perm[t, i] = row,
//   x_perm[row] = x[perm[row]].
//
// Stable ranks come from warp-level matching: __match_any_sync groups the lanes of a warp
// that hold the same expert, the rank inside the warp is the popcount of lower matching
// lanes, and per-warp counts are prefix-summed in warp order.  Assignments are processed in
// their natural order a = t * k + i, which is ascending t inside each expert.
//
// Small problems (T*k <= 1024) run as ONE CTA that does counting, prefix sums, positions and
// the row copy.  Larger ones run count -> scan -> scatter over 256-assignment tiles, then a
// grid-wide 16-byte row gather.
#include <mutex>
#include <string>

#include "common.cuh"

namespace zmoe {
namespace {

constexpr int kSmallMax = 1024;   // assignments handled by the single-CTA path
constexpr int kTile = 256;        // assignments per CTA in the multi-CTA path
constexpr int kMaxE = 64;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Reads and validates the expert of assignment a (-1 when out of range or a >= n).
__device__ __forceinline__ int load_expert(const int32_t* __restrict__ idx, int a, int n, int E, unsigned int* err) {
  if (a >= n) return -1;
  int e = idx[a];
  if (e < 0 || e >= E) {
    record_device_error(err);
    return -1;
  }
  return e;
}

// Copies row `src` of x to row `dst` of x_perm: `vecs` 16-byte vectors, one warp.
__device__ __forceinline__ void copy_row(const uint4* __restrict__ x, uint4* __restrict__ xp, int src, int dst,
                                         int vecs, int lane) {
  const uint4* s = x + static_cast<size_t>(src) * vecs;
  uint4* d = xp + static_cast<size_t>(dst) * vecs;
  for (int v = lane; v < vecs; v += 32) d[v] = s[v];
}

// ------------------------------------------------------------------------------------------
// single CTA: T*k <= 1024, blockDim.x = 1024
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) permute_small_kernel(
    const int32_t* __restrict__ idx, const uint4* __restrict__ x, int n, int k, int E, int vecs,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv_perm, uint4* __restrict__ x_perm, unsigned int* err) {
  __shared__ int wcnt[32][kMaxE];
  __shared__ int off_s[kMaxE + 1];
  __shared__ int rowsrc[kSmallMax];
  const int a = threadIdx.x;
  const int lane = a & 31, warp = a >> 5;
  for (int i = threadIdx.x; i < 32 * kMaxE; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int e = load_expert(idx, a, n, E, err);
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & lanemask_lt());
  if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < E) {
    int c = 0;
    for (int w = 0; w < 32; ++w) c += wcnt[w][threadIdx.x];
    off_s[threadIdx.x + 1] = c;   // temporarily the count
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    off_s[0] = 0;
    for (int i = 0; i < E; ++i) off_s[i + 1] += off_s[i];
  }
  __syncthreads();
  if (threadIdx.x < E) {
    const int ee = threadIdx.x;
    counts[ee] = off_s[ee + 1] - off_s[ee];
    int run = off_s[ee];
    for (int w = 0; w < 32; ++w) {
      const int c = wcnt[w][ee];
      wcnt[w][ee] = run;
      run += c;
    }
  }
  if (threadIdx.x <= E) offsets[threadIdx.x] = off_s[threadIdx.x];
  __syncthreads();
  if (a < n) {
    if (e >= 0) {
      const int pos = wcnt[warp][e] + rank;
      perm[pos] = a / k;
      inv_perm[a] = pos;
      rowsrc[pos] = a / k;
    } else {
      inv_perm[a] = -1;
    }
  }
  __syncthreads();
  const int rows = off_s[E];
  for (int r = warp; r < rows; r += 32) copy_row(x, x_perm, rowsrc[r], r, vecs, lane);
}

// ------------------------------------------------------------------------------------------
// multi CTA: tiles of 256 assignments
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kTile) permute_count_kernel(const int32_t* __restrict__ idx, int n, int E,
                                                                int32_t* __restrict__ tile_cnt, unsigned int* err) {
  __shared__ int hist[kMaxE];
  if (threadIdx.x < E) hist[threadIdx.x] = 0;
  __syncthreads();
  const int e = load_expert(idx, blockIdx.x * kTile + threadIdx.x, n, E, err);
  if (e >= 0) atomicAdd(&hist[e], 1);
  __syncthreads();
  if (threadIdx.x < E) tile_cnt[blockIdx.x * E + threadIdx.x] = hist[threadIdx.x];
}

// One CTA: totals, offsets, and each tile's base row per expert (in place over tile_cnt).
__global__ void permute_scan_kernel(int32_t* __restrict__ tile_cnt, int tiles, int E, int32_t* __restrict__ counts,
                                    int32_t* __restrict__ offsets) {
  __shared__ int tot[kMaxE + 1];
  const int e = threadIdx.x;
  if (e < E) {
    int c = 0;
    for (int b = 0; b < tiles; ++b) c += tile_cnt[b * E + e];
    tot[e + 1] = c;
    counts[e] = c;
  }
  __syncthreads();
  if (e == 0) {
    tot[0] = 0;
    for (int i = 0; i < E; ++i) tot[i + 1] += tot[i];
  }
  __syncthreads();
  if (e <= E) offsets[e] = tot[e];
  if (e < E) {
    int run = tot[e];
    for (int b = 0; b < tiles; ++b) {
      const int c = tile_cnt[b * E + e];
      tile_cnt[b * E + e] = run;
      run += c;
    }
  }
}

__global__ void __launch_bounds__(kTile) permute_scatter_kernel(const int32_t* __restrict__ idx, int n, int k, int E,
                                                                  const int32_t* __restrict__ tile_base,
                                                                  int32_t* __restrict__ perm,
                                                                  int32_t* __restrict__ inv_perm) {
  __shared__ int wcnt[kTile / 32][kMaxE];
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kTile / 32) * kMaxE; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int a = blockIdx.x * kTile + threadIdx.x;
  const int e = load_expert(idx, a, n, E, nullptr);   // errors were counted by the count pass
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & lanemask_lt());
  if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
  __syncthreads();
  if (a >= n) return;
  if (e < 0) {
    inv_perm[a] = -1;
    return;
  }
  int pos = tile_base[blockIdx.x * E + e] + rank;
  for (int w = 0; w < warp; ++w) pos += wcnt[w][e];
  perm[pos] = a / k;
  inv_perm[a] = pos;
}

// x_perm[row] = x[perm[row]] for rows < offsets[E]; one 16-byte vector per thread-iteration.
__global__ void gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                                   const int32_t* __restrict__ offsets, int E, int vecs, uint4* __restrict__ x_perm) {
  const long long rows = offsets[E];
  const long long total = rows * vecs;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / vecs;
    const int v = static_cast<int>(i - r * vecs);
    x_perm[i] = x[static_cast<size_t>(perm[r]) * vecs + v];
  }
}

int tiles_for(long long n) { return static_cast<int>((n + kTile - 1) / kTile); }

}  // namespace

// The index half of zmoe_permute (counts, offsets, perm, inv_perm; no row copy), for callers that move
// the rows themselves (the fp8 path quantizes them on the way).  Workspace as zmoe_permute's.
zmoe_status permute_indices(const int32_t* expert_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv_perm, void* workspace, size_t ws_bytes, cudaStream_t s) {
  const long long n = static_cast<long long>(T) * k;
  if (n <= 0) return ZMOE_OK;
  const int tiles = tiles_for(n);
  if (!workspace || ws_bytes < static_cast<size_t>(tiles) * E * sizeof(int32_t))
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL, "permute (indices): workspace too small");
  int32_t* tile_cnt = static_cast<int32_t*>(workspace);
  unsigned int* err = device_error_counter();
  permute_count_kernel<<<tiles, kTile, 0, s>>>(expert_idx, static_cast<int>(n), E, tile_cnt, err);
  permute_scan_kernel<<<1, 128, 0, s>>>(tile_cnt, tiles, E, counts, offsets);
  permute_scatter_kernel<<<tiles, kTile, 0, s>>>(expert_idx, static_cast<int>(n), k, E, tile_cnt, perm, inv_perm);
  return check_launch("permute (indices)");
}

}  // namespace zmoe

extern "C" {

size_t zmoe_permute_workspace_size(int T, int E, int k) {
  if (T < 0 || E < 1 || k < 1) return 0;
  const long long n = static_cast<long long>(T) * k;
  const long long tiles = (n + zmoe::kTile - 1) / zmoe::kTile;
  return static_cast<size_t>((tiles < 1 ? 1 : tiles) * E * sizeof(int32_t));
}

zmoe_status zmoe_permute(const int32_t* expert_idx, const void* x, zmoe_dtype dtype, int T, int d, int E, int k,
                         int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* x_perm,
                         void* workspace, size_t ws_bytes, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_permute");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(dtype), "zmoe_permute: bad dtype");
  ZMOE_REQUIRE(T >= 0, "zmoe_permute: T must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= kMaxE, "zmoe_permute: E must be in [1, 64]");
  ZMOE_REQUIRE(k == 1 || k == 2, "zmoe_permute: k must be 1 or 2");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0, "zmoe_permute: d must be a positive multiple of 8");
  ZMOE_REQUIRE(counts && offsets, "zmoe_permute: counts/offsets NULL");
  const long long n = static_cast<long long>(T) * k;
  ZMOE_REQUIRE(n <= 0x7fffffffLL, "zmoe_permute: T * k overflows int32");
  if (n > 0) {
    ZMOE_REQUIRE(expert_idx && x && perm && inv_perm && x_perm, "zmoe_permute: NULL pointer");
    ZMOE_REQUIRE(aligned16(x) && aligned16(x_perm), "zmoe_permute: x/x_perm not 16-byte aligned");
  }
  const int vecs = static_cast<int>(d * dtype_size(dtype) / 16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = device_error_counter();
  clear_error();
  if (n <= kSmallMax) {
    permute_small_kernel<<<1, 1024, 0, s>>>(expert_idx, static_cast<const uint4*>(x), static_cast<int>(n), k, E, vecs,
                                            counts, offsets, perm, inv_perm, static_cast<uint4*>(x_perm), err);
    return check_launch("zmoe_permute");
  }
  const int tiles = tiles_for(n);
  const size_t need = static_cast<size_t>(tiles) * E * sizeof(int32_t);
  if (!workspace || ws_bytes < need)
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL, "zmoe_permute: workspace smaller than zmoe_permute_workspace_size()");
  int32_t* tile_cnt = static_cast<int32_t*>(workspace);
  permute_count_kernel<<<tiles, kTile, 0, s>>>(expert_idx, static_cast<int>(n), E, tile_cnt, err);
  permute_scan_kernel<<<1, 128, 0, s>>>(tile_cnt, tiles, E, counts, offsets);
  permute_scatter_kernel<<<tiles, kTile, 0, s>>>(expert_idx, static_cast<int>(n), k, E, tile_cnt, perm, inv_perm);
  const long long total_vecs = n * vecs;
  long long grid = (total_vecs + 255) / 256;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (grid > cap) grid = cap;
  gather_rows_kernel<<<static_cast<int>(grid), 256, 0, s>>>(static_cast<const uint4*>(x), perm, offsets, E, vecs,
                                                            static_cast<uint4*>(x_perm));
  return check_launch("zmoe_permute");
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// zmoe_permute_noalloc: the same permutation for callers that cannot allocate device memory.
//
// The multi-CTA path keeps per-tile expert counts in scratch.  Here that scratch is a
// file-scope device array, so the call allocates nothing: every GPU that loads this library
// holds the array (64 KB) until the process exits.  In host code `g_noalloc_tile_counts` is
// only a host-side stand-in for the symbol, never a device address; its device address is
// fetched with cudaGetSymbolAddress once per device, with that device current, on the first
// call made on that device, and cached for the life of the process (a device reset after that
// first call is not supported).  Every call shares the array and it keeps the last call's
// contents: the count pass writes every entry the later passes read, so nothing needs clearing,
// but two calls that overlap on the GPU (different streams, no ordering) race on it.
// ---------------------------------------------------------------------------------------------
namespace zmoe {
namespace {

constexpr int kNoAllocMaxTiles = 256;   // 256 tiles x 256 assignments = 65536 assignments
static __device__ __align__(256) int32_t g_noalloc_tile_counts[kNoAllocMaxTiles * kMaxE];

std::mutex g_noalloc_mutex;
int32_t* g_noalloc_addr[64] = {};

// Device address of the static scratch on the current device (set up once per device).
zmoe_status noalloc_scratch(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(ZMOE_ERR_CUDA, std::string("zmoe_permute_noalloc: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(ZMOE_ERR_UNSUPPORTED, "zmoe_permute_noalloc: device index >= 64");
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    int32_t* ptr = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_tile_counts);
    if (e != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();   // consume the error so that a later call's launch check does not report it
      return fail(ZMOE_ERR_CUDA, std::string("zmoe_permute_noalloc: cudaGetSymbolAddress failed: ") +
                                     cudaGetErrorString(e));
    }
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return ZMOE_OK;
}

}  // namespace
}  // namespace zmoe

extern "C" zmoe_status zmoe_permute_noalloc(const int32_t* expert_idx, const void* x, zmoe_dtype dtype, int T, int d,
                                            int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm,
                                            int32_t* inv_perm, void* x_perm, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_permute_noalloc");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(dtype), "zmoe_permute_noalloc: bad dtype");
  ZMOE_REQUIRE(T >= 0, "zmoe_permute_noalloc: T must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= kMaxE, "zmoe_permute_noalloc: E must be in [1, 64]");
  ZMOE_REQUIRE(k == 1 || k == 2, "zmoe_permute_noalloc: k must be 1 or 2");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0, "zmoe_permute_noalloc: d must be a positive multiple of 8");
  ZMOE_REQUIRE(counts && offsets, "zmoe_permute_noalloc: counts/offsets NULL");
  const long long n = static_cast<long long>(T) * k;
  ZMOE_REQUIRE(n <= static_cast<long long>(kNoAllocMaxTiles) * kTile,
               "zmoe_permute_noalloc: T * k exceeds the 65536 assignments its static scratch holds; "
               "use zmoe_permute with a caller-provided workspace");
  if (n > 0) {
    ZMOE_REQUIRE(expert_idx && x && perm && inv_perm && x_perm, "zmoe_permute_noalloc: NULL pointer");
    ZMOE_REQUIRE(aligned16(x) && aligned16(x_perm), "zmoe_permute_noalloc: x/x_perm not 16-byte aligned");
  }
  const int vecs = static_cast<int>(d * dtype_size(dtype) / 16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = device_error_counter();
  clear_error();
  if (n <= kSmallMax) {
    permute_small_kernel<<<1, 1024, 0, s>>>(expert_idx, static_cast<const uint4*>(x), static_cast<int>(n), k, E, vecs,
                                            counts, offsets, perm, inv_perm, static_cast<uint4*>(x_perm), err);
    return check_launch("zmoe_permute_noalloc");
  }
  int32_t* tile_cnt = nullptr;
  zmoe_status st = noalloc_scratch(&tile_cnt);
  if (st != ZMOE_OK) return st;
  const int tiles = tiles_for(n);
  permute_count_kernel<<<tiles, kTile, 0, s>>>(expert_idx, static_cast<int>(n), E, tile_cnt, err);
  permute_scan_kernel<<<1, 128, 0, s>>>(tile_cnt, tiles, E, counts, offsets);
  permute_scatter_kernel<<<tiles, kTile, 0, s>>>(expert_idx, static_cast<int>(n), k, E, tile_cnt, perm, inv_perm);
  const long long total_vecs = n * vecs;
  long long grid = (total_vecs + 255) / 256;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (grid > cap) grid = cap;
  gather_rows_kernel<<<static_cast<int>(grid), 256, 0, s>>>(static_cast<const uint4*>(x), perm, offsets, E, vecs,
                                                            static_cast<uint4*>(x_perm));
  return check_launch("zmoe_permute_noalloc");
}
