// Embedding-gradient scatter-add that allocates nothing: the sort and chunk
// scratch of the deterministic scatter (scatter.cu) lives in one fixed-size
// array in device memory that the library defines at file scope.
//
// Some callers cannot allocate device memory at the point where they need
// this gradient: code whose device memory is all handed out by a host
// framework's pool (a plug-in op inside another runtime, a server that
// reserves its whole memory budget up front), where a cudaMalloc would either
// fail or be forbidden, and which cannot size a gpt_config workspace either.
// They pass only the inputs and the output; the library supplies the scratch.
//
// The array is loaded on every GPU that loads this library and stays resident
// until the process exits.  Its device address belongs to a CUDA context, so
// it is looked up on the first call made in each context (keyed by the
// context's unique id, which a context created after cudaDeviceReset, or by
// the driver API inside a host runtime, does not share with an earlier one).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "device_common.cuh"

namespace gpt {

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxContexts = 64;

__device__ __align__(256) unsigned char g_scatter_scratch[kScratchBytes];

// device address of g_scatter_scratch per context (unique id), most recent
// contexts kept when more than kMaxContexts have called
struct ScratchAddr {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_addr_mu;
ScratchAddr g_addr[kMaxContexts] = {};
int g_addr_next = 0;

uint64_t up256(uint64_t x) { return (x + 255) / 256 * 256; }

// Scratch regions of the sort + scatter for N tokens, vocabulary V and width
// d, at 256-byte aligned offsets from the scratch base; returns the bytes used.
uint64_t scratch_layout(int64_t N, int64_t V, int64_t d, Layout* L) {
  uint64_t off = 0;
  auto take = [&](uint64_t bytes) {
    off = up256(off);
    uint64_t o = off;
    off += bytes;
    return o;
  };
  L->N = N;
  L->sort_tiles = (N + 1023) / 1024;
  L->sort_perm = take(N * 4);
  L->sort_offs = take((V + 1) * 4);
  L->sort_count = take((V + 1) * 4);
  L->sort_tilehist = take(uint64_t(L->sort_tiles) * V * 4);
  L->scat_max_items = N / 64 + V + 1;
  L->scat_items = take(uint64_t(L->scat_max_items) * 8);
  L->scat_item_offs = take((V + 1) * 8);
  L->scat_partial = take(uint64_t(N / 64 + 1) * d * 4 * 2);
  return up256(off);
}

// Unique id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array in the current context.  The first
// call in a context looks it up (cudaGetSymbolAddress, with that context
// current); later calls reuse it.  Without a readable context id the address
// is looked up on every call.
int scratch_address(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPT_ECUDA;
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (id)
    for (const ScratchAddr& a : g_addr)
      if (a.ctx_id == id) {
        *out = static_cast<char*>(a.addr);
        return GPT_OK;
      }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scatter_scratch) != cudaSuccess || !p) return GPT_ECUDA;
  if (id) {
    g_addr[g_addr_next] = {id, p};
    g_addr_next = (g_addr_next + 1) % kMaxContexts;
  }
  *out = static_cast<char*>(p);
  return GPT_OK;
}

}  // namespace
}  // namespace gpt

extern "C" int gpt_embedding_grad_noalloc(const int32_t* tokens, int64_t n_tokens, int32_t vocab,
                                          int32_t d_model, int32_t dtype, const float* dx0,
                                          void* dwte, int accumulate, void* stream) {
  using namespace gpt;
  if (!tokens || !dx0 || !dwte || n_tokens <= 0 || vocab < 2 || d_model <= 0)
    return GPT_EINVAL;
  if (dtype != GPT_BF16 && dtype != GPT_F32) return GPT_EINVAL;
  if (accumulate != 0 && accumulate != 1) return GPT_EINVAL;
  if ((reinterpret_cast<uintptr_t>(tokens) | reinterpret_cast<uintptr_t>(dx0) |
       reinterpret_cast<uintptr_t>(dwte)) % 16)
    return GPT_EINVAL;
  if (n_tokens > (int64_t(1) << 24) || vocab > (1 << 24)) return GPT_EUNSUPPORTED;
  Layout L{};
  if (scratch_layout(n_tokens, vocab, d_model, &L) > kScratchBytes) return GPT_EUNSUPPORTED;
  char* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc) return rc;
  gpt_config c{};
  c.vocab = vocab;
  c.d_model = d_model;
  c.dtype = dtype;
  c.batch = 1;
  c.seq_len = int32_t(n_tokens);
  if (launch_sort_tokens(c, L, tokens, scratch, stream)) return GPT_ECUDA;
  if (launch_embed_scatter(c, L, dx0, scratch, dwte, accumulate, stream)) return GPT_ECUDA;
  return GPT_OK;
}
