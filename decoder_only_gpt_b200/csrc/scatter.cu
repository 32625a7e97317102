// Deterministic embedding-gradient scatter-add:
//   dwte[v] = sum over positions n with tokens[n] == v of dx0[n]   (fp32 sum -> storage)
//
// 1. Stable counting sort of positions by token id (integer work, bit-exact
//    with a CPU stable sort):
//      counts[v] and per-tile counts tilehist[tile][v] (integer atomics: the
//      totals do not depend on order); exclusive scan -> offs[v]; column-wise
//      prefix over tiles -> each tile's first slot per token; inside a tile of
//      1024 positions a bitonic sort of (token, position) keys gives each
//      position its rank among equal tokens.
// 2. Work items = (row v, chunk j) with chunks of 64 consecutive sorted
//    positions.  A row with one chunk is summed and stored directly; a row
//    with several (the Zipf head: id 0 takes ~14 % of positions) stores
//    per-chunk partials that a second kernel adds in chunk order.  Every sum
//    runs in a fixed order, so the result is bit-identical across runs.
#include "device_common.cuh"

namespace gpt {

constexpr int kSortTile = 1024;
constexpr int kChunk = 64;

__global__ void histogram_kernel(const int32_t* __restrict__ tok, int64_t N, int V,
                                 int32_t* __restrict__ counts, int32_t* __restrict__ tilehist) {
  int64_t n = int64_t(blockIdx.x) * kSortTile + threadIdx.x;
  if (n >= N) return;
  int t = tok[n];
  if (t < 0 || t >= V) t = 0;  // out-of-range ids were reported by the gather
  atomicAdd(&counts[t], 1);
  atomicAdd(&tilehist[int64_t(blockIdx.x) * V + t], 1);
}

// Exclusive scan of `n` int2 values (x and y scanned independently) by one block.
// out[n] receives the totals.
__global__ void scan2_kernel(const int2* __restrict__ in, int2* __restrict__ out, int n) {
  __shared__ int2 warp_tot[32];
  __shared__ int2 carry;
  if (threadIdx.x == 0) carry = make_int2(0, 0);
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int base = 0; base < n; base += blockDim.x) {
    int i = base + threadIdx.x;
    int2 v = i < n ? in[i] : make_int2(0, 0);
    int2 incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int ax = __shfl_up_sync(0xffffffffu, incl.x, o);
      int ay = __shfl_up_sync(0xffffffffu, incl.y, o);
      if (lane >= o) { incl.x += ax; incl.y += ay; }
    }
    if (lane == 31) warp_tot[w] = incl;
    __syncthreads();
    if (w == 0) {
      int2 t = lane < int(blockDim.x >> 5) ? warp_tot[lane] : make_int2(0, 0);
      int2 ti = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int ax = __shfl_up_sync(0xffffffffu, ti.x, o);
        int ay = __shfl_up_sync(0xffffffffu, ti.y, o);
        if (lane >= o) { ti.x += ax; ti.y += ay; }
      }
      warp_tot[lane] = make_int2(ti.x - t.x, ti.y - t.y);  // exclusive warp offsets
    }
    __syncthreads();
    int2 c = carry;
    int2 wo = warp_tot[w];
    if (i < n) out[i] = make_int2(c.x + wo.x + incl.x - v.x, c.y + wo.y + incl.y - v.y);
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1)
      carry = make_int2(c.x + wo.x + incl.x, c.y + wo.y + incl.y);
    __syncthreads();
  }
  if (threadIdx.x == 0) out[n] = carry;
}

// counts -> int2(count, 0) so the pair scan can be reused
__global__ void pack_counts_kernel(const int32_t* __restrict__ counts, int2* __restrict__ pair,
                                   int V) {
  int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v < V) pair[v] = make_int2(counts[v], 0);
}

__global__ void unpack_offs_kernel(const int2* __restrict__ pair, int32_t* __restrict__ offs,
                                   int V) {
  int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v <= V) offs[v] = pair[v].x;
}

// tilehist[tile][v] <- offs[v] + sum_{tile' < tile} tilehist[tile'][v]
__global__ void tile_prefix_kernel(int32_t* __restrict__ tilehist, const int32_t* __restrict__ offs,
                                   int tiles, int V) {
  int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= V) return;
  int run = offs[v];
  for (int t = 0; t < tiles; ++t) {
    int c = tilehist[int64_t(t) * V + v];
    tilehist[int64_t(t) * V + v] = run;
    run += c;
  }
}

__global__ void __launch_bounds__(kSortTile) place_kernel(const int32_t* __restrict__ tok,
                                                          int64_t N, int V,
                                                          const int32_t* __restrict__ tilebase,
                                                          int32_t* __restrict__ perm) {
  __shared__ unsigned long long key[kSortTile];
  __shared__ int head[kSortTile];
  const int tid = threadIdx.x;
  const int64_t n = int64_t(blockIdx.x) * kSortTile + tid;
  unsigned long long k = ~0ull;
  if (n < N) {
    int t = tok[n];
    if (t < 0 || t >= V) t = 0;
    k = (static_cast<unsigned long long>(t) << 10) | unsigned(tid);
  }
  key[tid] = k;
  __syncthreads();
  // bitonic sort, ascending
  for (int size = 2; size <= kSortTile; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      int partner = tid ^ stride;
      if (partner > tid) {
        unsigned long long a = key[tid], b = key[partner];
        bool up = (tid & size) == 0;
        if ((a > b) == up) { key[tid] = b; key[partner] = a; }
      }
      __syncthreads();
    }
  }
  unsigned long long mine = key[tid];
  bool valid = mine != ~0ull;
  int my_tok = int(mine >> 10);
  bool is_head = tid == 0 || (key[tid - 1] >> 10) != (mine >> 10);
  head[tid] = is_head ? tid : 0;
  __syncthreads();
  // inclusive max-scan of head indices (Hillis-Steele)
  for (int o = 1; o < kSortTile; o <<= 1) {
    int v = head[tid];
    int u = tid >= o ? head[tid - o] : 0;
    __syncthreads();
    head[tid] = max(v, u);
    __syncthreads();
  }
  if (valid) {
    int rank = tid - head[tid];
    int local = int(mine & 1023ull);
    int dst = tilebase[int64_t(blockIdx.x) * V + my_tok] + rank;
    perm[dst] = int(int64_t(blockIdx.x) * kSortTile + local);
  }
}

int launch_sort_tokens(const gpt_config& c, const Layout& L, const int32_t* tok, char* ws,
                       void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  const int V = c.vocab;
  const int64_t N = L.N;
  const int tiles = int(L.sort_tiles);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.sort_count);
  int32_t* tilehist = reinterpret_cast<int32_t*>(ws + L.sort_tilehist);
  int32_t* offs = reinterpret_cast<int32_t*>(ws + L.sort_offs);
  int32_t* perm = reinterpret_cast<int32_t*>(ws + L.sort_perm);
  int2* pair_in = reinterpret_cast<int2*>(ws + L.scat_items);  // scratch, reused later
  int2* pair_out = reinterpret_cast<int2*>(ws + L.scat_item_offs);
  if (cudaMemsetAsync(counts, 0, size_t(V + 1) * 4, st) != cudaSuccess) return 1;
  if (cudaMemsetAsync(tilehist, 0, size_t(tiles) * V * 4, st) != cudaSuccess) return 1;
  histogram_kernel<<<tiles, kSortTile, 0, st>>>(tok, N, V, counts, tilehist);
  pack_counts_kernel<<<ceil_div(V, 256), 256, 0, st>>>(counts, pair_in, V);
  scan2_kernel<<<1, 1024, 0, st>>>(pair_in, pair_out, V);
  unpack_offs_kernel<<<ceil_div(V + 1, 256), 256, 0, st>>>(pair_out, offs, V);
  tile_prefix_kernel<<<ceil_div(V, 256), 256, 0, st>>>(tilehist, offs, tiles, V);
  place_kernel<<<tiles, kSortTile, 0, st>>>(tok, N, V, tilehist, perm);
  return last_launch_rc();
}

// ---------------------------------------------------------------------------
// scatter
// ---------------------------------------------------------------------------
// pair[v] = (chunks of row v, chunks of row v if it has more than one else 0)
__global__ void chunk_count_kernel(const int32_t* __restrict__ offs, int2* __restrict__ pair,
                                   int V) {
  int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= V) return;
  int cnt = offs[v + 1] - offs[v];
  int ch = (cnt + kChunk - 1) / kChunk;
  pair[v] = make_int2(ch, ch > 1 ? ch : 0);
}

// item list: items[item_offs[v] + j] = (v, j)
__global__ void fill_items_kernel(const int2* __restrict__ ioffs, int2* __restrict__ items,
                                  int V) {
  int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= V) return;
  int b = ioffs[v].x, e = ioffs[v + 1].x;
  for (int j = 0; j < e - b; ++j) items[b + j] = make_int2(v, j);
}

template <typename T>
__global__ void chunk_sum_kernel(const int2* __restrict__ items, const int2* __restrict__ ioffs,
                                 const int32_t* __restrict__ offs, const int32_t* __restrict__ perm,
                                 const float* __restrict__ dx0, int d, int V,
                                 float* __restrict__ partial, T* __restrict__ dwte,
                                 int accumulate) {
  const int total = ioffs[V].x;
  const int item = blockIdx.x;
  if (item >= total) return;
  const int2 it = items[item];
  const int v = it.x, j = it.y;
  const int beg = offs[v] + j * kChunk;
  const int end = min(offs[v + 1], beg + kChunk);
  const int nch = ioffs[v + 1].x - ioffs[v].x;
  for (int col = threadIdx.x; col < d; col += blockDim.x) {
    float s = 0.f;
    for (int p = beg; p < end; ++p) s += dx0[int64_t(perm[p]) * d + col];
    if (nch == 1) {
      T* dst = dwte + int64_t(v) * d + col;
      *dst = from_f<T>(accumulate ? to_f(*dst) + s : s);
    } else {
      partial[int64_t(ioffs[v].y + j) * d + col] = s;
    }
  }
}

// rows with several chunks: add the partials in chunk order; rows without any
// position: zero (unless accumulating)
template <typename T>
__global__ void row_finish_kernel(const int2* __restrict__ ioffs, const float* __restrict__ partial,
                                  int d, T* __restrict__ dwte, int accumulate) {
  const int v = blockIdx.x;
  const int nch = ioffs[v + 1].x - ioffs[v].x;
  if (nch == 1) return;
  T* row = dwte + int64_t(v) * d;
  if (nch == 0) {
    if (!accumulate)
      for (int col = threadIdx.x; col < d; col += blockDim.x) row[col] = from_f<T>(0.f);
    return;
  }
  const int base = ioffs[v].y;
  for (int col = threadIdx.x; col < d; col += blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < nch; ++j) s += partial[int64_t(base + j) * d + col];
    row[col] = from_f<T>(accumulate ? to_f(row[col]) + s : s);
  }
}

int launch_embed_scatter(const gpt_config& c, const Layout& L, const float* dx0, char* ws,
                         void* dwte, int accumulate, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  const int V = c.vocab, d = c.d_model;
  const int32_t* offs = reinterpret_cast<const int32_t*>(ws + L.sort_offs);
  const int32_t* perm = reinterpret_cast<const int32_t*>(ws + L.sort_perm);
  int2* pair = reinterpret_cast<int2*>(ws + L.scat_items);  // scratch before the item list
  int2* ioffs = reinterpret_cast<int2*>(ws + L.scat_item_offs);
  int2* items = reinterpret_cast<int2*>(ws + L.scat_items);
  float* partial = reinterpret_cast<float*>(ws + L.scat_partial);
  chunk_count_kernel<<<ceil_div(V, 256), 256, 0, st>>>(offs, pair, V);
  scan2_kernel<<<1, 1024, 0, st>>>(pair, ioffs, V);
  fill_items_kernel<<<ceil_div(V, 256), 256, 0, st>>>(ioffs, items, V);
  const int max_items = int(L.scat_max_items);
  const int threads = d >= 512 ? 256 : 128;
  if (c.dtype == GPT_BF16) {
    chunk_sum_kernel<__nv_bfloat16><<<max_items, threads, 0, st>>>(
        items, ioffs, offs, perm, dx0, d, V, partial, (__nv_bfloat16*)dwte, accumulate);
    row_finish_kernel<__nv_bfloat16><<<V, threads, 0, st>>>(ioffs, partial, d,
                                                            (__nv_bfloat16*)dwte, accumulate);
  } else {
    chunk_sum_kernel<float><<<max_items, threads, 0, st>>>(items, ioffs, offs, perm, dx0, d, V,
                                                          partial, (float*)dwte, accumulate);
    row_finish_kernel<float><<<V, threads, 0, st>>>(ioffs, partial, d, (float*)dwte,
                                                    accumulate);
  }
  return last_launch_rc();
}

}  // namespace gpt
