// ulysses_attn_bwd_noalloc: the attention backward for callers that cannot
// allocate device memory. Its scratch (per row: lse*log2(e) and D_i) lives in a
// fixed file-scope device array instead of a caller-supplied workspace.
#include <mutex>

#include "kernels.h"
#include "ulysses.h"

namespace uly {
namespace noalloc {

// Scratch for the backward's prep kernel output: 32 MiB, 256-byte aligned.
// Every GPU that loads this library holds it until the process exits.
constexpr size_t kScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// The array's device address on the current device, looked up once per device.
// (In host code `g_bwd_scratch` names a host-side shadow, not device memory.)
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace noalloc
}  // namespace uly

extern "C" uly_status ulysses_attn_bwd_noalloc(
    const void* const* q_head, const void* const* k_head, const void* const* v_head, const void* const* o_head,
    const float* const* lse_head, const void* const* do_head, void* const* dq_head, void* const* dk_head,
    void* const* dv_head, int64_t N, int P, int H, int H_kv, int d, const int32_t* cu_seqlens, int num_seqs,
    int max_seqlen, float softmax_scale, int rank_lo, int rank_hi, cudaStream_t stream) {
  // The shape check first, so a shape that ulysses_attn_bwd rejects gets the
  // same status here (INVALID_ARG or UNSUPPORTED), before the size test.
  const uly_status st = check_shape(N, P, H, H_kv, d, rank_lo, rank_hi);
  if (st != ULY_OK) return st;
  const size_t need = ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, 1);
  if (need == 0) return ULY_ERR_INVALID_ARG;
  if (need > uly::noalloc::kScratchBytes) return ULY_ERR_UNSUPPORTED;  // beyond the fixed scratch
  void* scratch = nullptr;
  if (uly::noalloc::scratch_address(&scratch) != cudaSuccess) return ULY_ERR_CUDA;
  return ulysses_attn_bwd(q_head, k_head, v_head, o_head, lse_head, do_head, dq_head, dk_head, dv_head, N, P, H,
                          H_kv, d, cu_seqlens, num_seqs, max_seqlen, softmax_scale, 1, scratch,
                          uly::noalloc::kScratchBytes, rank_lo, rank_hi, stream);
}
