// Embedding-backward entry point that allocates nothing.
//
// Some callers cannot allocate device memory when they call into this
// library: code running inside a CUDA-graph capture or an allocator hook,
// plug-ins whose host framework owns every allocation, or real-time loops
// that forbid cudaMalloc after start-up.  For them the scratch of the
// embedding backward (the stable radix sort of token ids and the row
// offsets) lives in a file-scope __device__ array instead of caller memory.
//
// The array is a fixed 1.5 MiB per GPU that loads the library, held until the
// process exits.  Host code must not use the array's name as a device
// address (on the host it names a stand-in object): the device address is
// looked up once per device with cudaGetSymbolAddress and cached.
#include <mutex>

#include "../../include/llm.h"
#include "../../include/llm_kernels.h"
#include "internal.h"

namespace {

constexpr int64_t kMaxTokens = 65536;
constexpr int kMaxVocab = 65536;
// int32 words the embedding backward needs at the maximum sizes: keys and
// positions twice (ping-pong of the radix sort), 256 digit counters per
// 256-token block, vocab+1 row offsets, the count and list of the runs longer
// than 64 rows (at most tokens / 64 of them), and slack.
constexpr int64_t kScratchInts = 4 * kMaxTokens + 256 * (kMaxTokens / 256) + (kMaxVocab + 1) + 1 +
                                 (kMaxTokens / 64 + 1) + 64;

static __device__ __align__(256) int32_t g_embed_bwd_scratch[kScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t *g_scratch_dev_ptr[kMaxDevices] = {};

}  // namespace

extern "C" int llm_kernel_embed_bwd_noalloc(const int32_t *d_tokens, const float *d_dx,
                                            float *d_dwte, int64_t n_tokens, int d_model,
                                            int vocab, void *stream) {
  if (!d_tokens || !d_dx || !d_dwte || n_tokens < 1 || d_model < 1 || vocab < 1)
    return LLM_ERR_ARG;
  if (n_tokens > kMaxTokens || vocab > kMaxVocab) return LLM_ERR_ARG;
  if (llm::embed_bwd_scratch_ints(n_tokens, vocab) > kScratchInts) return LLM_ERR_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LLM_ERR_CUDA;
  int32_t *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_dev_ptr[dev]) {
      // First call on this device (which is current): resolve the array's
      // device address.
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_embed_bwd_scratch) != cudaSuccess || !p)
        return LLM_ERR_CUDA;
      g_scratch_dev_ptr[dev] = (int32_t *)p;
    }
    scratch = g_scratch_dev_ptr[dev];
  }
  llm::embed_bwd(d_tokens, d_dx, d_dwte, n_tokens, d_model, vocab, scratch, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}
