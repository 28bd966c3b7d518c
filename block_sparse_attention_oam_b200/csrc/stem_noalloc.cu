// stem_attention_noalloc: the whole prefill path with its scratch memory taken
// from a fixed array compiled into this library instead of a caller workspace.
//
// Some callers cannot allocate device memory at all: plugin or custom-operator
// hosts whose framework owns every byte of the GPU through its own allocator,
// and serving loops that must not allocate once they are running.  They can still
// pass their inputs and outputs; this entry point needs nothing else.
#include <mutex>

#include "stem_internal.cuh"

namespace stem {
namespace {

// Scratch for the pooled summaries, the packed scores, the CSR selection and the
// status word.  It exists once per device that loads the library, for the life of
// the process, and every call on that device shares it.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

}  // namespace
}  // namespace stem

using namespace stem;

extern "C" STEM_API stem_status_t stem_attention_noalloc(const stem_problem_t* prob, const void* q, const void* k,
                                                         const void* v, const stem_paged_kv_t* paged, void* out,
                                                         float* lse, int32_t* row_ptr_out, int32_t* col_idx_out,
                                                         uint32_t* status_out, void* stream) {
  // size check first: a problem that does not fit is refused before any CUDA call
  stem_sizes_t sz;
  const stem_status_t vs = stem_query_sizes(prob, &sz);
  if (vs != STEM_OK) return vs;
  if (sz.workspace_bytes > kStaticScratchBytes)
    return set_last_error(STEM_ERR_WORKSPACE,
                          "stem_attention_noalloc: this problem needs %zu bytes of scratch but the static scratch "
                          "holds %zu; use stem_attention with a caller workspace",
                          sz.workspace_bytes, kStaticScratchBytes);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return set_last_error(STEM_ERR_CUDA, "stem_attention_noalloc: no usable current device");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (g_addr[dev] == nullptr) {
      // host code cannot use g_scratch directly: its name is a host-side shadow,
      // not a device address.  The device address is looked up once per device and
      // kept for the life of the process; a device reset (cudaDeviceReset, or a
      // destroyed and recreated primary context) reloads the module and leaves the
      // kept address stale, so this entry point must not be used across one.
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
      if (e != cudaSuccess || p == nullptr)
        return set_last_error(STEM_ERR_CUDA, "stem_attention_noalloc: scratch address lookup failed: %s",
                              cudaGetErrorString(e));
      g_addr[dev] = p;
    }
    scratch = g_addr[dev];
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word is the only part of the scratch that must start at zero
  if (cudaMemsetAsync(scratch, 0, 256, st) != cudaSuccess)
    return set_last_error(STEM_ERR_CUDA, "stem_attention_noalloc: clearing the status word failed");
  stem_status_t s = stem_attention(prob, q, k, v, paged, out, lse, row_ptr_out, col_idx_out, scratch,
                                   kStaticScratchBytes, stream);
  if (s != STEM_OK) return s;
  if (status_out != nullptr &&
      cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return set_last_error(STEM_ERR_CUDA, "stem_attention_noalloc: copying the status word failed");
  return STEM_OK;
}
