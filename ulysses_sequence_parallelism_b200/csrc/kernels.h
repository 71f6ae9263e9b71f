// Host-side launchers shared between the C-ABI layer (api.cu) and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace uly {

struct AttnShape {
  int N;          // tokens (all ranks)
  int P;          // virtual ranks
  int Hl;         // query heads per rank (H/P)
  int Hkvl;       // key/value heads per rank (H_kv/P)
  int d;          // head dim
  const int32_t* cu_seqlens;   // device, or null
  int num_seqs;
  float scale;    // softmax scale (already resolved; > 0)
  int rank_lo, rank_hi;
};

int permute_max_row_vecs();
cudaError_t launch_permute(bool seq_to_head, const void* const* src[3], void* const* dst[3], const int hx[3],
                           int64_t N, int P, int d, int rank_lo, int rank_hi, cudaStream_t stream);
// One head fragment per slot: global heads [f_lo[s], f_lo[s] + f_cnt[s]) of
// tensor s between the P sequence shards and the single head-side buffer at
// index 0 of the head-side pointer array ([N, f_cnt[s], d]).
cudaError_t launch_permute_fragment(bool seq_to_head, const void* const* src[3], void* const* dst[3],
                                    const int hx[3], const int f_lo[3], const int f_cnt[3], int64_t N, int P, int d,
                                    cudaStream_t stream);

// Pack (one rank's sequence shard -> per-destination chunks [P][N/P][f][d]) or
// unpack (the inverse) of head chunk [lo[s], lo[s] + f[s]) inside every rank's
// hx[s]/P heads, for up to three tensors (null src/dst: slot unused).
int exchange_max_row_vecs();
cudaError_t launch_exchange(bool pack, const void* const src[3], void* const dst[3], const int hx[3],
                            const int lo[3], const int f[3], int64_t N, int P, int d, cudaStream_t stream);

cudaError_t launch_attn_fwd(const AttnShape& s, const void* const* q, const void* const* k,
                            const void* const* v, void* const* o, float* const* lse, cudaStream_t stream);

// The same kernels reading Q/K/V (and dO, O) straight from the sequence shards
// and writing O (and dQ, dK, dV) straight into them: the permutes disappear.
cudaError_t launch_attn_fwd_seq(const AttnShape& s, const void* const* q_seq, const void* const* k_seq,
                                const void* const* v_seq, void* const* o_seq, float* const* lse, cudaStream_t stream);
cudaError_t launch_attn_bwd_seq(const AttnShape& s, const void* const* q_seq, const void* const* k_seq,
                                const void* const* v_seq, const void* const* o_seq, const float* const* lse,
                                const void* const* do_seq, void* const* dq_seq, void* const* dk_seq,
                                void* const* dv_seq, void* workspace, size_t workspace_bytes, int deterministic,
                                cudaStream_t stream);

// deterministic == 0 with d == 128 selects the one-pass backward (fp32 dQ
// accumulator in the workspace); everything else runs the two-pass kernels.
size_t attn_bwd_workspace_bytes(int64_t N, int P, int Hl, int d, int deterministic);
// The sequence-layout backward's workspace: the above plus, for the one-pass
// kernel, head-sharded copies of Q and dO (staged by a permute, since the
// kernel streams them faster from head shards than from sequence shards).
size_t attn_bwd_seq_workspace_bytes(int64_t N, int P, int Hl, int d, int deterministic);
// Whether the one-pass kernel's shared-memory layout fits when its dynamic
// shared memory starts dyn_base_offset bytes into the CTA's shared window.
bool attn_bwd_onepass_layout_fits(uint32_t dyn_base_offset);
cudaError_t launch_attn_bwd(const AttnShape& s, const void* const* q, const void* const* k,
                            const void* const* v, const void* const* o, const float* const* lse,
                            const void* const* dO, void* const* dq, void* const* dk, void* const* dv,
                            void* workspace, int deterministic, cudaStream_t stream);

// One projection GEMM (C = A B^T over a reduction of K, bf16 in, fp32
// accumulate, bf16 out) with operand views that fold the Ulysses all-to-alls
// into its loads and stores. Sources (proj_sm100.cu, enum Src): 0 SEQ_K,
// 1 HEAD_K, 2 PLAIN_K, 3 PLAIN_MN, 4 SEQ_MN, 5 HEAD_MN; outputs: 0 head shards,
// 1 sequence shards, 2 plain row-major bf16 matrix, 3 plain row-major fp32
// matrix added into (split-K chunks of k_chunk reduction elements).
struct ProjGemm {
  int a_src, b_src, out_kind, tok_m;
  int k_chunk;
  const void* const* a_bufs[3];   // per tensor: P head shards, or P sequence shards ([0]), or {matrix} ([0][0])
  int a_ntensors;
  int64_t a_plain_rows, a_plain_cols, a_seq_cols;
  const void* const* b_bufs[3];
  int b_ntensors;
  int64_t b_plain_rows, b_plain_cols, b_seq_cols;
  void* out[3][16];               // per tensor and rank / shard, or out[0][0]
  int64_t N;
  int P, K, n_out, m_rows, H, H_kv, d;
};
cudaError_t launch_proj_gemm(const ProjGemm& g, cudaStream_t stream);

}  // namespace uly
