// C-ABI entry points: argument validation, then the kernel launchers.
// Nothing here allocates, frees or synchronises device memory except
// ulysses_get_device_status / ulysses_set_wait_limit, which touch the
// library's own device words.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "ulysses.h"

namespace uly {
// Waits (bounded) on an mbarrier that nothing ever arrives on: exercises the
// same give-up path as the attention kernels, without touching a real workload.
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(b, 0, 0x7Fu, 0xABC);
}
}  // namespace uly

namespace {

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uly_status check_shape(int64_t N, int P, int H, int H_kv, int d, int rank_lo, int rank_hi) {
  if (P < 1 || N <= 0 || H <= 0 || H_kv <= 0) return ULY_ERR_INVALID_ARG;
  if (P > ULY_MAX_RANKS) return ULY_ERR_UNSUPPORTED;
  if (N % P != 0 || H % P != 0 || H_kv % P != 0 || H % H_kv != 0) return ULY_ERR_INVALID_ARG;
  if (rank_lo < 0 || rank_hi > P || rank_lo >= rank_hi) return ULY_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ULY_ERR_UNSUPPORTED;
  if (N > INT32_MAX || (N / P) * static_cast<int64_t>(H) * d >= (int64_t(1) << 31) ||
      N * static_cast<int64_t>(H / P) * d >= (int64_t(1) << 31))
    return ULY_ERR_UNSUPPORTED;
  return ULY_OK;
}

// Every entry of ranks [lo, hi) must be a 16-byte aligned non-null pointer.
bool ranks_ok(const void* const* arr, int lo, int hi) {
  if (arr == nullptr) return false;
  for (int r = lo; r < hi; ++r)
    if (!aligned16(arr[r])) return false;
  return true;
}

uly_status from_cuda(cudaError_t e) { return e == cudaSuccess ? ULY_OK : ULY_ERR_CUDA; }

uly_status check_cu(const int32_t* cu, int num_seqs, int64_t N) {
  if (cu == nullptr) return ULY_OK;
  if (num_seqs < 1 || num_seqs > N) return ULY_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return ULY_ERR_INVALID_ARG;
  return ULY_OK;
}

uly_status a2a(bool seq_to_head, const void* const* s0, const void* const* s1, const void* const* s2,
               void* const* d0, void* const* d1, void* const* d2, int64_t N, int P, int H, int H_kv, int d,
               const int32_t* cu, int num_seqs, int rank_lo, int rank_hi, cudaStream_t stream) {
  uly_status st = check_shape(N, P, H, H_kv, d, rank_lo, rank_hi);
  if (st != ULY_OK) return st;
  if (check_cu(cu, num_seqs, N) != ULY_OK) return ULY_ERR_INVALID_ARG;
  if (s0 == nullptr || d0 == nullptr) return ULY_ERR_INVALID_ARG;
  if ((s1 == nullptr) != (d1 == nullptr) || (s2 == nullptr) != (d2 == nullptr)) return ULY_ERR_INVALID_ARG;
  if (H * (d / 8) > uly::permute_max_row_vecs()) return ULY_ERR_UNSUPPORTED;
  // Sequence side: every rank. Head side: ranks in range.
  const void* const* src[3] = {s0, s1, s2};
  void* const* dst[3] = {d0, d1, d2};
  for (int s = 0; s < 3; ++s) {
    if (src[s] == nullptr) continue;
    const int slo = seq_to_head ? 0 : rank_lo, shi = seq_to_head ? P : rank_hi;
    const int dlo = seq_to_head ? rank_lo : 0, dhi = seq_to_head ? rank_hi : P;
    if (!ranks_ok(src[s], slo, shi) || !ranks_ok(reinterpret_cast<const void* const*>(dst[s]), dlo, dhi))
      return ULY_ERR_INVALID_ARG;
  }
  const int hx[3] = {H, H_kv, H_kv};
  return from_cuda(uly::launch_permute(seq_to_head, src, dst, hx, N, P, d, rank_lo, rank_hi, stream));
}

// A head fragment: whole GQA groups inside one rank's query heads.
uly_status check_fragment(int64_t N, int P, int H, int H_kv, int d, int head_lo, int num_heads) {
  uly_status st = check_shape(N, P, H, H_kv, d, 0, P);
  if (st != ULY_OK) return st;
  const int group = H / H_kv, hl = H / P;
  if (num_heads < 1 || head_lo < 0 || head_lo + num_heads > H) return ULY_ERR_INVALID_ARG;
  if (head_lo % group != 0 || num_heads % group != 0) return ULY_ERR_INVALID_ARG;
  if (head_lo / hl != (head_lo + num_heads - 1) / hl) return ULY_ERR_INVALID_ARG;   // inside one rank
  return ULY_OK;
}

uly_status a2a_fragment(bool seq_to_head, const void* const* seq0, const void* const* seq1,
                        const void* const* seq2, const void* f0, const void* f1, const void* f2, int64_t N, int P,
                        int H, int H_kv, int d, int head_lo, int num_heads, cudaStream_t stream) {
  uly_status st = check_fragment(N, P, H, H_kv, d, head_lo, num_heads);
  if (st != ULY_OK) return st;
  if (seq0 == nullptr || f0 == nullptr) return ULY_ERR_INVALID_ARG;
  if ((seq1 == nullptr) != (f1 == nullptr) || (seq2 == nullptr) != (f2 == nullptr)) return ULY_ERR_INVALID_ARG;
  if (H * (d / 8) > uly::permute_max_row_vecs()) return ULY_ERR_UNSUPPORTED;
  const void* const* seq[3] = {seq0, seq1, seq2};
  const void* frag[3] = {f0, f1, f2};
  const void* fptr[3][1] = {{f0}, {f1}, {f2}};
  for (int s = 0; s < 3; ++s) {
    if (seq[s] == nullptr) continue;
    if (!ranks_ok(seq[s], 0, P) || !aligned16(frag[s])) return ULY_ERR_INVALID_ARG;
  }
  const int group = H / H_kv;
  const int hx[3] = {H, H_kv, H_kv};
  const int f_lo[3] = {head_lo, head_lo / group, head_lo / group};
  const int f_cnt[3] = {num_heads, num_heads / group, num_heads / group};
  const void* const* head[3] = {fptr[0], fptr[1], fptr[2]};
  const void* const* src[3];
  void* const* dst[3];
  for (int s = 0; s < 3; ++s) {
    const bool on = seq[s] != nullptr;
    src[s] = !on ? nullptr : (seq_to_head ? seq[s] : head[s]);
    dst[s] = !on ? nullptr : const_cast<void* const*>(seq_to_head ? head[s] : seq[s]);
  }
  return from_cuda(uly::launch_permute_fragment(seq_to_head, src, dst, hx, f_lo, f_cnt, N, P, d, stream));
}

// Pack/unpack for the multi-process exchange: one rank's shards and its
// [P][N/P][f][d] chunk buffers; the head chunk is whole GQA groups.
uly_status exchange(bool pack, const void* s0, const void* s1, const void* s2, void* d0, void* d1, void* d2,
                    int64_t N, int P, int H, int H_kv, int d, int head_lo, int num_heads, cudaStream_t stream) {
  uly_status st = check_shape(N, P, H, H_kv, d, 0, P);
  if (st != ULY_OK) return st;
  const int group = H / H_kv, hl = H / P;
  if (num_heads < 1 || head_lo < 0 || head_lo + num_heads > hl) return ULY_ERR_INVALID_ARG;
  if (head_lo % group != 0 || num_heads % group != 0) return ULY_ERR_INVALID_ARG;
  if (s0 == nullptr || d0 == nullptr) return ULY_ERR_INVALID_ARG;
  if ((s1 == nullptr) != (d1 == nullptr) || (s2 == nullptr) != (d2 == nullptr)) return ULY_ERR_INVALID_ARG;
  const void* src[3] = {s0, s1, s2};
  void* dst[3] = {d0, d1, d2};
  for (int k = 0; k < 3; ++k)
    if (src[k] != nullptr && (!aligned16(src[k]) || !aligned16(dst[k]))) return ULY_ERR_INVALID_ARG;
  if (H * (d / 8) > uly::exchange_max_row_vecs()) return ULY_ERR_UNSUPPORTED;
  const int hx[3] = {H, H_kv, H_kv};
  const int lo[3] = {head_lo, head_lo / group, head_lo / group};
  const int f[3] = {num_heads, num_heads / group, num_heads / group};
  return from_cuda(uly::launch_exchange(pack, src, dst, hx, lo, f, N, P, d, stream));
}

// Token chunk of the split-K weight-gradient GEMMs. Measured at 64K tokens
// (Llama shapes): the output-projection backward takes 7.00 / 6.34 / 6.02 /
// 5.86 / 5.77 / 5.78 / 6.28 ms with chunks of 1K / 2K / 4K / 8K / 16K / 32K /
// 64K tokens: longer chunks spread each CTA's pipeline fill and fp32 epilogue
// over more MMAs, until too few CTAs remain to fill the GPU evenly.
constexpr int kProjTokenChunk = 16384;

uly_status check_proj(int64_t N, int P, int H, int H_kv, int d, int hidden) {
  uly_status st = check_shape(N, P, H, H_kv, d, 0, P);
  if (st != ULY_OK) return st;
  if (hidden <= 0) return ULY_ERR_INVALID_ARG;
  if ((N / P) % 128 != 0 || hidden % 256 != 0 || ((H + 2 * H_kv) * d) % 256 != 0) return ULY_ERR_UNSUPPORTED;
  if ((N / P) * static_cast<int64_t>(hidden) >= (int64_t(1) << 31)) return ULY_ERR_UNSUPPORTED;
  return ULY_OK;
}

float resolve_scale(float softmax_scale, int d) {
  return (softmax_scale > 0.f && isfinite(softmax_scale)) ? softmax_scale : 1.0f / sqrtf(static_cast<float>(d));
}

}  // namespace

extern "C" {

uly_status ulysses_a2a_seq_to_head(const void* const* x0_seq, const void* const* x1_seq, const void* const* x2_seq,
                                   void* const* x0_head, void* const* x1_head, void* const* x2_head, int64_t N,
                                   int P, int H, int H_kv, int d, const int32_t* cu_seqlens, int num_seqs,
                                   int rank_lo, int rank_hi, cudaStream_t stream) {
  return a2a(true, x0_seq, x1_seq, x2_seq, x0_head, x1_head, x2_head, N, P, H, H_kv, d, cu_seqlens, num_seqs,
             rank_lo, rank_hi, stream);
}

uly_status ulysses_a2a_head_to_seq(const void* const* x0_head, const void* const* x1_head,
                                   const void* const* x2_head, void* const* x0_seq, void* const* x1_seq,
                                   void* const* x2_seq, int64_t N, int P, int H, int H_kv, int d,
                                   const int32_t* cu_seqlens, int num_seqs, int rank_lo, int rank_hi,
                                   cudaStream_t stream) {
  return a2a(false, x0_head, x1_head, x2_head, x0_seq, x1_seq, x2_seq, N, P, H, H_kv, d, cu_seqlens, num_seqs,
             rank_lo, rank_hi, stream);
}

uly_status ulysses_a2a_seq_to_head_frag(const void* const* x0_seq, const void* const* x1_seq,
                                        const void* const* x2_seq, void* x0_frag, void* x1_frag, void* x2_frag,
                                        int64_t N, int P, int H, int H_kv, int d, int head_lo, int num_heads,
                                        cudaStream_t stream) {
  return a2a_fragment(true, x0_seq, x1_seq, x2_seq, x0_frag, x1_frag, x2_frag, N, P, H, H_kv, d, head_lo, num_heads,
                      stream);
}

uly_status ulysses_a2a_head_to_seq_frag(const void* x0_frag, const void* x1_frag, const void* x2_frag,
                                        void* const* x0_seq, void* const* x1_seq, void* const* x2_seq, int64_t N,
                                        int P, int H, int H_kv, int d, int head_lo, int num_heads,
                                        cudaStream_t stream) {
  auto cv = [](void* const* p) { return reinterpret_cast<const void* const*>(p); };
  return a2a_fragment(false, cv(x0_seq), cv(x1_seq), cv(x2_seq), x0_frag, x1_frag, x2_frag, N, P, H, H_kv, d,
                      head_lo, num_heads, stream);
}

uly_status ulysses_a2a_pack(const void* x0_seq, const void* x1_seq, const void* x2_seq, void* x0_send,
                            void* x1_send, void* x2_send, int64_t N, int P, int H, int H_kv, int d, int head_lo,
                            int num_heads, cudaStream_t stream) {
  return exchange(true, x0_seq, x1_seq, x2_seq, x0_send, x1_send, x2_send, N, P, H, H_kv, d, head_lo, num_heads,
                  stream);
}

uly_status ulysses_a2a_unpack(const void* x0_recv, const void* x1_recv, const void* x2_recv, void* x0_seq,
                              void* x1_seq, void* x2_seq, int64_t N, int P, int H, int H_kv, int d, int head_lo,
                              int num_heads, cudaStream_t stream) {
  return exchange(false, x0_recv, x1_recv, x2_recv, x0_seq, x1_seq, x2_seq, N, P, H, H_kv, d, head_lo, num_heads,
                  stream);
}

uly_status ulysses_qkv_proj_seq_to_head(const void* const* x_seq, const void* w_qkv, void* const* q_head,
                                        void* const* k_head, void* const* v_head, int64_t N, int P, int H,
                                        int H_kv, int d, int hidden, cudaStream_t stream) {
  uly_status st = check_proj(N, P, H, H_kv, d, hidden);
  if (st != ULY_OK) return st;
  auto cv = [](void* const* p) { return reinterpret_cast<const void* const*>(p); };
  if (!ranks_ok(x_seq, 0, P) || !aligned16(w_qkv) || !ranks_ok(cv(q_head), 0, P) || !ranks_ok(cv(k_head), 0, P) ||
      !ranks_ok(cv(v_head), 0, P))
    return ULY_ERR_INVALID_ARG;
  const void* wq[1] = {w_qkv};
  uly::ProjGemm g{};
  g.a_src = 0; g.b_src = 2; g.out_kind = 0; g.tok_m = 1;
  g.a_bufs[0] = x_seq; g.a_ntensors = 1; g.a_seq_cols = hidden;
  g.b_bufs[0] = wq; g.b_ntensors = 1; g.b_plain_rows = (H + 2 * H_kv) * d; g.b_plain_cols = hidden;
  for (int r = 0; r < P; ++r) { g.out[0][r] = q_head[r]; g.out[1][r] = k_head[r]; g.out[2][r] = v_head[r]; }
  g.N = N; g.P = P; g.K = hidden; g.n_out = (H + 2 * H_kv) * d; g.H = H; g.H_kv = H_kv; g.d = d;
  return from_cuda(uly::launch_proj_gemm(g, stream));
}

uly_status ulysses_out_proj_head_to_seq(const void* const* o_head, const void* w_o, void* const* y_seq, int64_t N,
                                        int P, int H, int H_kv, int d, int hidden, cudaStream_t stream) {
  uly_status st = check_proj(N, P, H, H_kv, d, hidden);
  if (st != ULY_OK) return st;
  if (!ranks_ok(o_head, 0, P) || !aligned16(w_o) || !ranks_ok(reinterpret_cast<const void* const*>(y_seq), 0, P))
    return ULY_ERR_INVALID_ARG;
  const void* wo[1] = {w_o};
  uly::ProjGemm g{};
  g.a_src = 1; g.b_src = 2; g.out_kind = 1; g.tok_m = 1;
  g.a_bufs[0] = o_head; g.a_ntensors = 1;
  g.b_bufs[0] = wo; g.b_ntensors = 1; g.b_plain_rows = hidden; g.b_plain_cols = static_cast<int64_t>(H) * d;
  for (int r = 0; r < P; ++r) g.out[0][r] = y_seq[r];
  g.N = N; g.P = P; g.K = H * d; g.n_out = hidden; g.H = H; g.H_kv = H_kv; g.d = d;
  return from_cuda(uly::launch_proj_gemm(g, stream));
}

uly_status ulysses_out_proj_bwd(const void* const* o_head, const void* w_o, const void* const* dy_seq,
                                void* const* do_head, void* dw_o, int64_t N, int P, int H, int H_kv, int d,
                                int hidden, cudaStream_t stream) {
  uly_status st = check_proj(N, P, H, H_kv, d, hidden);
  if (st != ULY_OK) return st;
  if ((H * d) % 256 != 0) return ULY_ERR_UNSUPPORTED;
  if (!ranks_ok(o_head, 0, P) || !aligned16(w_o) || !ranks_ok(dy_seq, 0, P) ||
      !ranks_ok(reinterpret_cast<const void* const*>(do_head), 0, P) || !aligned16(dw_o))
    return ULY_ERR_INVALID_ARG;
  const void* wo[1] = {w_o};
  // dO = dY W_o, written into the head shards
  uly::ProjGemm g{};
  g.a_src = 0; g.b_src = 3; g.out_kind = 0; g.tok_m = 1;
  g.a_bufs[0] = dy_seq; g.a_ntensors = 1; g.a_seq_cols = hidden;
  g.b_bufs[0] = wo; g.b_ntensors = 1; g.b_plain_rows = hidden; g.b_plain_cols = static_cast<int64_t>(H) * d;
  for (int r = 0; r < P; ++r) g.out[0][r] = do_head[r];
  g.N = N; g.P = P; g.K = hidden; g.n_out = H * d; g.H = H; g.H_kv = H_kv; g.d = d;
  cudaError_t e = uly::launch_proj_gemm(g, stream);
  if (e != cudaSuccess) return from_cuda(e);
  // dW_o = dY^T O (fp32), O read from the head shards; split over token chunks
  e = cudaMemsetAsync(dw_o, 0, static_cast<size_t>(hidden) * H * d * sizeof(float), stream);
  if (e != cudaSuccess) return from_cuda(e);
  uly::ProjGemm w{};
  w.a_src = 4; w.b_src = 5; w.out_kind = 3; w.tok_m = 0; w.k_chunk = kProjTokenChunk;
  w.a_bufs[0] = dy_seq; w.a_ntensors = 1; w.a_seq_cols = hidden;
  w.b_bufs[0] = o_head; w.b_ntensors = 1;
  w.out[0][0] = dw_o;
  w.N = N; w.P = P; w.K = static_cast<int>(N); w.n_out = H * d; w.m_rows = hidden; w.H = H; w.H_kv = H_kv; w.d = d;
  return from_cuda(uly::launch_proj_gemm(w, stream));
}

uly_status ulysses_qkv_proj_bwd(const void* const* x_seq, const void* w_qkv, const void* const* dq_head,
                                const void* const* dk_head, const void* const* dv_head, void* const* dx_seq,
                                void* dw_qkv, int64_t N, int P, int H, int H_kv, int d, int hidden,
                                cudaStream_t stream) {
  uly_status st = check_proj(N, P, H, H_kv, d, hidden);
  if (st != ULY_OK) return st;
  if (!ranks_ok(x_seq, 0, P) || !aligned16(w_qkv) || !ranks_ok(dq_head, 0, P) || !ranks_ok(dk_head, 0, P) ||
      !ranks_ok(dv_head, 0, P) || !ranks_ok(reinterpret_cast<const void* const*>(dx_seq), 0, P) ||
      !aligned16(dw_qkv))
    return ULY_ERR_INVALID_ARG;
  const void* wq[1] = {w_qkv};
  const int n_feat = (H + 2 * H_kv) * d;
  // dX = [dQ|dK|dV] W_qkv, gathered from the head shards, written into the sequence shards
  uly::ProjGemm g{};
  g.a_src = 1; g.b_src = 3; g.out_kind = 1; g.tok_m = 1;
  g.a_bufs[0] = dq_head; g.a_bufs[1] = dk_head; g.a_bufs[2] = dv_head; g.a_ntensors = 3;
  g.b_bufs[0] = wq; g.b_ntensors = 1; g.b_plain_rows = n_feat; g.b_plain_cols = hidden;
  for (int r = 0; r < P; ++r) g.out[0][r] = dx_seq[r];
  g.N = N; g.P = P; g.K = n_feat; g.n_out = hidden; g.H = H; g.H_kv = H_kv; g.d = d;
  cudaError_t e = uly::launch_proj_gemm(g, stream);
  if (e != cudaSuccess) return from_cuda(e);
  // dW_qkv = [dQ|dK|dV]^T X (fp32); split over token chunks
  e = cudaMemsetAsync(dw_qkv, 0, static_cast<size_t>(n_feat) * hidden * sizeof(float), stream);
  if (e != cudaSuccess) return from_cuda(e);
  uly::ProjGemm w{};
  w.a_src = 5; w.b_src = 4; w.out_kind = 3; w.tok_m = 0; w.k_chunk = kProjTokenChunk;
  w.a_bufs[0] = dq_head; w.a_bufs[1] = dk_head; w.a_bufs[2] = dv_head; w.a_ntensors = 3;
  w.b_bufs[0] = x_seq; w.b_ntensors = 1; w.b_seq_cols = hidden;
  w.out[0][0] = dw_qkv;
  w.N = N; w.P = P; w.K = static_cast<int>(N); w.n_out = hidden; w.m_rows = n_feat; w.H = H; w.H_kv = H_kv;
  w.d = d;
  return from_cuda(uly::launch_proj_gemm(w, stream));
}

uly_status ulysses_attn_fwd(const void* const* q_head, const void* const* k_head, const void* const* v_head,
                            void* const* o_head, float* const* lse_head, int64_t N, int P, int H, int H_kv, int d,
                            const int32_t* cu_seqlens, int num_seqs, int max_seqlen, float softmax_scale,
                            int causal, int rank_lo, int rank_hi, cudaStream_t stream) {
  (void)max_seqlen;
  uly_status st = check_shape(N, P, H, H_kv, d, rank_lo, rank_hi);
  if (st != ULY_OK) return st;
  if (causal != 1) return ULY_ERR_UNSUPPORTED;
  if (check_cu(cu_seqlens, num_seqs, N) != ULY_OK) return ULY_ERR_INVALID_ARG;
  if (!ranks_ok(q_head, rank_lo, rank_hi) || !ranks_ok(k_head, rank_lo, rank_hi) ||
      !ranks_ok(v_head, rank_lo, rank_hi) || !ranks_ok(reinterpret_cast<const void* const*>(o_head), rank_lo, rank_hi) ||
      !ranks_ok(reinterpret_cast<const void* const*>(lse_head), rank_lo, rank_hi))
    return ULY_ERR_INVALID_ARG;
  uly::AttnShape s{static_cast<int>(N), P, H / P, H_kv / P, d, cu_seqlens, cu_seqlens ? num_seqs : 1,
                   resolve_scale(softmax_scale, d), rank_lo, rank_hi};
  return from_cuda(uly::launch_attn_fwd(s, q_head, k_head, v_head, o_head, lse_head, stream));
}

size_t ulysses_attn_bwd_workspace_size(int64_t N, int P, int H, int H_kv, int d, int deterministic) {
  if (check_shape(N, P, H, H_kv, d, 0, P > 0 ? P : 1) != ULY_OK) return 0;
  return uly::attn_bwd_workspace_bytes(N, P, H / P, d, deterministic);
}

uly_status ulysses_attn_bwd(const void* const* q_head, const void* const* k_head, const void* const* v_head,
                            const void* const* o_head, const float* const* lse_head, const void* const* do_head,
                            void* const* dq_head, void* const* dk_head, void* const* dv_head, int64_t N, int P,
                            int H, int H_kv, int d, const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
                            float softmax_scale, int deterministic, void* workspace, size_t workspace_bytes,
                            int rank_lo, int rank_hi, cudaStream_t stream) {
  (void)max_seqlen;
  uly_status st = check_shape(N, P, H, H_kv, d, rank_lo, rank_hi);
  if (st != ULY_OK) return st;
  if (check_cu(cu_seqlens, num_seqs, N) != ULY_OK) return ULY_ERR_INVALID_ARG;
  auto cv = [](void* const* p) { return reinterpret_cast<const void* const*>(p); };
  if (!ranks_ok(q_head, rank_lo, rank_hi) || !ranks_ok(k_head, rank_lo, rank_hi) ||
      !ranks_ok(v_head, rank_lo, rank_hi) || !ranks_ok(o_head, rank_lo, rank_hi) ||
      !ranks_ok(reinterpret_cast<const void* const*>(lse_head), rank_lo, rank_hi) ||
      !ranks_ok(do_head, rank_lo, rank_hi) || !ranks_ok(cv(dq_head), rank_lo, rank_hi) ||
      !ranks_ok(cv(dk_head), rank_lo, rank_hi) || !ranks_ok(cv(dv_head), rank_lo, rank_hi))
    return ULY_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ULY_ERR_INVALID_ARG;
  if (workspace_bytes < uly::attn_bwd_workspace_bytes(N, P, H / P, d, deterministic)) return ULY_ERR_INVALID_ARG;
  uly::AttnShape s{static_cast<int>(N), P, H / P, H_kv / P, d, cu_seqlens, cu_seqlens ? num_seqs : 1,
                   resolve_scale(softmax_scale, d), rank_lo, rank_hi};
  return from_cuda(uly::launch_attn_bwd(s, q_head, k_head, v_head, o_head, lse_head, do_head, dq_head, dk_head,
                                        dv_head, workspace, deterministic, stream));
}

uly_status ulysses_attn_fwd_seq(const void* const* q_seq, const void* const* k_seq, const void* const* v_seq,
                                void* const* o_seq, float* const* lse_head, int64_t N, int P, int H, int H_kv,
                                int d, const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
                                float softmax_scale, int causal, int rank_lo, int rank_hi, cudaStream_t stream) {
  (void)max_seqlen;
  uly_status st = check_shape(N, P, H, H_kv, d, rank_lo, rank_hi);
  if (st != ULY_OK) return st;
  if (causal != 1 || (N / P) % 128 != 0) return ULY_ERR_UNSUPPORTED;
  if (check_cu(cu_seqlens, num_seqs, N) != ULY_OK) return ULY_ERR_INVALID_ARG;
  if (!ranks_ok(q_seq, 0, P) || !ranks_ok(k_seq, 0, P) || !ranks_ok(v_seq, 0, P) ||
      !ranks_ok(reinterpret_cast<const void* const*>(o_seq), 0, P) ||
      !ranks_ok(reinterpret_cast<const void* const*>(lse_head), rank_lo, rank_hi))
    return ULY_ERR_INVALID_ARG;
  uly::AttnShape s{static_cast<int>(N), P, H / P, H_kv / P, d, cu_seqlens, cu_seqlens ? num_seqs : 1,
                   resolve_scale(softmax_scale, d), rank_lo, rank_hi};
  return from_cuda(uly::launch_attn_fwd_seq(s, q_seq, k_seq, v_seq, o_seq, lse_head, stream));
}

uly_status ulysses_attn_bwd_seq(const void* const* q_seq, const void* const* k_seq, const void* const* v_seq,
                                const void* const* o_seq, const float* const* lse_head, const void* const* do_seq,
                                void* const* dq_seq, void* const* dk_seq, void* const* dv_seq, int64_t N, int P,
                                int H, int H_kv, int d, const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
                                float softmax_scale, int deterministic, void* workspace,
                                size_t workspace_bytes, int rank_lo, int rank_hi, cudaStream_t stream) {
  (void)max_seqlen;
  uly_status st = check_shape(N, P, H, H_kv, d, rank_lo, rank_hi);
  if (st != ULY_OK) return st;
  if ((N / P) % 128 != 0) return ULY_ERR_UNSUPPORTED;
  if (check_cu(cu_seqlens, num_seqs, N) != ULY_OK) return ULY_ERR_INVALID_ARG;
  auto cv = [](void* const* p) { return reinterpret_cast<const void* const*>(p); };
  if (!ranks_ok(q_seq, 0, P) || !ranks_ok(k_seq, 0, P) || !ranks_ok(v_seq, 0, P) || !ranks_ok(o_seq, 0, P) ||
      !ranks_ok(do_seq, 0, P) || !ranks_ok(cv(dq_seq), 0, P) || !ranks_ok(cv(dk_seq), 0, P) ||
      !ranks_ok(cv(dv_seq), 0, P) ||
      !ranks_ok(reinterpret_cast<const void* const*>(lse_head), rank_lo, rank_hi))
    return ULY_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ULY_ERR_INVALID_ARG;
  if (workspace_bytes < uly::attn_bwd_workspace_bytes(N, P, H / P, d, deterministic)) return ULY_ERR_INVALID_ARG;
  uly::AttnShape s{static_cast<int>(N), P, H / P, H_kv / P, d, cu_seqlens, cu_seqlens ? num_seqs : 1,
                   resolve_scale(softmax_scale, d), rank_lo, rank_hi};
  return from_cuda(uly::launch_attn_bwd_seq(s, q_seq, k_seq, v_seq, o_seq, lse_head, do_seq, dq_seq, dk_seq,
                                            dv_seq, workspace, workspace_bytes, deterministic, stream));
}

size_t ulysses_attn_bwd_seq_workspace_size(int64_t N, int P, int H, int H_kv, int d, int deterministic) {
  if (check_shape(N, P, H, H_kv, d, 0, P > 0 ? P : 1) != ULY_OK) return 0;
  return uly::attn_bwd_seq_workspace_bytes(N, P, H / P, d, deterministic);
}

const char* ulysses_status_string(uly_status s) {
  switch (s) {
    case ULY_OK: return "ok";
    case ULY_ERR_INVALID_ARG: return "invalid argument";
    case ULY_ERR_UNSUPPORTED: return "unsupported shape or option";
    case ULY_ERR_CUDA: return "CUDA runtime error";
    case ULY_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

uly_status ulysses_get_device_status(cudaStream_t stream, uint32_t* detail) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ULY_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpyFromSymbol(&w, uly::g_error_word, sizeof(w)) != cudaSuccess) return ULY_ERR_CUDA;
  const uint32_t zero = 0;
  if (w != 0 && cudaMemcpyToSymbol(uly::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return ULY_ERR_CUDA;
  if (detail) *detail = w;
  return w == 0 ? ULY_OK : ULY_ERR_TIMEOUT;
}

void ulysses_set_wait_limit(uint32_t iters) { cudaMemcpyToSymbol(uly::g_wait_limit, &iters, sizeof(iters)); }

int ulysses_attn_bwd_onepass_layout_fits(uint32_t dyn_smem_offset) {
  return uly::attn_bwd_onepass_layout_fits(dyn_smem_offset) ? 1 : 0;
}

uly_status ulysses_selftest_bounded_wait(cudaStream_t stream) {
  uly::selftest_wait_kernel<<<1, 32, 0, stream>>>();
  return from_cuda(cudaGetLastError());
}

}  // extern "C"
