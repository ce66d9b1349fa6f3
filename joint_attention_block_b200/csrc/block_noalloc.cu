// dit_block_forward for callers that cannot allocate device memory.
//
// Some hosts never allocate device memory after start-up: engines that reserve
// all of it up front, plugin interfaces that hand a kernel only its input and
// output buffers with no allocator, and latency-critical paths where a
// cudaMalloc (which may synchronise the device) is not acceptable.  Such a
// caller cannot provide the workspace dit_block_forward asks for, so this entry
// point runs the same block forward with its scratch in a fixed array that the
// library itself holds in device memory.
//
// The array below is sized once for every GPU that loads this library and lives
// until the process exits.  Host code cannot use the array's name as a device
// address (it names a host-side stand-in), so the first call on each device,
// with that device current, asks the runtime for the array's device address and
// keeps it.  Nothing here allocates.
#include <mutex>

#include "internal.h"
#include "jab_dit.h"

namespace {

static_assert(DIT_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

// Scratch of the no-allocation entry point: intermediates of one block forward
// (rotary tables, normalised activations, q/k/v, attention output, residual,
// MLP hidden).  Shared by every call; it keeps the last call's contents.
__device__ __align__(256) uint8_t g_noalloc_scratch[DIT_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_CUDA;
  if (dev < 0 || dev >= 64) return DIT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DIT_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DIT_OK;
}

}  // namespace

extern "C" int dit_block_forward_noalloc(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in,
                                          void* x_out, int batch, int n_text, int grid_h, int grid_w, int t_img,
                                          const int32_t* pos, void* stream) {
  const size_t need = dit_block_workspace_bytes(cfg, batch, n_text, grid_h, grid_w);
  if (need == 0) {
    // invalid or unsupported configuration: let the regular entry point say which
    return dit_block_forward(cfg, w, x_in, x_out, batch, n_text, grid_h, grid_w, t_img, pos, nullptr, 0, stream);
  }
  if (need > DIT_NOALLOC_SCRATCH_BYTES) return DIT_ERR_UNSUPPORTED;  // shape too large for the fixed scratch
  void* scratch = nullptr;
  const int st = noalloc_scratch(&scratch);
  if (st != DIT_OK) return st;
  // Every intermediate is written before it is read, so the scratch needs no clearing.
  return dit_block_forward(cfg, w, x_in, x_out, batch, n_text, grid_h, grid_w, t_img, pos, scratch,
                           DIT_NOALLOC_SCRATCH_BYTES, stream);
}
