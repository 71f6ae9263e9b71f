/*
 * ulysses.h -- C ABI of the single-GPU Ulysses sequence-parallel attention layer
 * for NVIDIA B200 (sm_100a).
 *
 * The layer (theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually
 * Work?"; radardeia.com, "Arquitetura Técnica"): every rank holds a contiguous
 * chunk of N/P tokens; an all-to-all turns that into all N positions for H/P
 * heads; each rank runs full-sequence causal attention on its heads (heads are
 * independent); the inverse all-to-all returns the output to sequence sharding.
 * Here the P ranks are P disjoint device buffers on one GPU, so each
 * all-to-all is an on-device permute.
 *
 * Layouts (all row-major, bf16 unless stated):
 *   sequence shard, rank p : [N/P, Hx, d]   token t = p*N/P + s
 *   head shard, rank p     : [N, Hx/P, d]   local head j = global head p*Hx/P + j
 *   LSE, rank p            : float32 [H/P, N] (natural log of the scaled scores' sum)
 *   Hx = H for Q, O, dO, dQ;  Hx = H_kv for K, V, dK, dV.
 *   Query head h reads key/value head h / (H/H_kv).
 *
 * Conventions for every entry point:
 *   - Rank buffers are passed as HOST arrays of P DEVICE pointers, indexed by
 *     rank. Entries of ranks outside [rank_lo, rank_hi) are not read and may
 *     be NULL. The caller owns all device memory (including workspace); the
 *     library never allocates or frees device memory.
 *   - Every device pointer must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream) and do
 *     not synchronise, except ulysses_get_device_status() and the host
 *     pipeline's synchronize/destroy (which run on the handle's own streams).
 *   - Arguments are validated before any launch. On ULY_ERR_INVALID_ARG or
 *     ULY_ERR_UNSUPPORTED nothing is launched and no memory is touched. A
 *     launch failure returns ULY_ERR_CUDA. Nothing aborts or traps.
 *   - Supported shapes: 1 <= P <= ULY_MAX_RANKS; N % P == 0; H % P == 0;
 *     H_kv % P == 0 (the pages require at least as many heads as ranks;
 *     strengthened here so that heads split evenly -- contenidos2-1ml.pages.dev,
 *     "¿Qué cambia en la práctica...?"); H % H_kv == 0; d in {64, 128}; N/P*H*d < 2^31.
 *   - cu_seqlens: DEVICE int32 array [num_seqs+1], cu_seqlens[0] = 0,
 *     non-decreasing, cu_seqlens[num_seqs] = N (packed variable-length
 *     documents, block-diagonal causal mask). NULL = one causal sequence.
 *     The kernels clamp what they read, so malformed contents give wrong
 *     numbers but never an out-of-bounds access.
 */
#ifndef ULYSSES_B200_H
#define ULYSSES_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ULY_MAX_RANKS 16

#if defined(__GNUC__)
#define ULY_API __attribute__((visibility("default")))
#else
#define ULY_API
#endif

typedef enum {
  ULY_OK = 0,
  ULY_ERR_INVALID_ARG = 1,   /* bad pointer, size, range or alignment */
  ULY_ERR_UNSUPPORTED = 2,   /* valid but not implemented (d, P, causal=0, ...) */
  ULY_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  ULY_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up (see get_device_status) */
} uly_status;

/* All-to-all #1, sequence sharding -> head sharding: afterwards each rank holds
 * the whole sequence for its subset of heads (theaicatchup.com, "How Does
 * Ulysses Sequence Parallelism Actually Work?").
 *   dst[q][t, j, :] = src[t / (N/P)][t % (N/P), q*Hx/P + j, :]
 * Up to three tensors move in one launch: slot 0 has H heads (Q, or dO in the
 * backward), slots 1 and 2 have H_kv heads (K, V). A NULL slot-1/2 array skips
 * that tensor. Only destination ranks q in [rank_lo, rank_hi) are written
 * (0..P for all); every source rank is read. cu_seqlens/num_seqs are accepted
 * for symmetry and ignored (the permute is a pure index map; documents may
 * straddle shards). Bit-exact copy. */
ULY_API uly_status ulysses_a2a_seq_to_head(
    const void* const* x0_seq, const void* const* x1_seq, const void* const* x2_seq,
    void* const* x0_head, void* const* x1_head, void* const* x2_head,
    int64_t N, int P, int H, int H_kv, int d,
    const int32_t* cu_seqlens, int num_seqs,
    int rank_lo, int rank_hi, cudaStream_t stream);

/* All-to-all #2, head sharding -> sequence sharding: the exact inverse of
 * ulysses_a2a_seq_to_head: after attention the first exchange is undone
 * (theaicatchup.com, ibid.; radardeia.com, "Arquitetura Técnica").
 *   dst[p][s, q*Hx/P + j, :] = src[q][p*N/P + s, j, :]
 * Slot 0: H heads (O; dQ in the backward); slots 1, 2: H_kv heads (dK, dV).
 * Only SOURCE ranks q in [rank_lo, rank_hi) are read, i.e. only their head
 * columns of every destination shard are written. Bit-exact copy. */
ULY_API uly_status ulysses_a2a_head_to_seq(
    const void* const* x0_head, const void* const* x1_head, const void* const* x2_head,
    void* const* x0_seq, void* const* x1_seq, void* const* x2_seq,
    int64_t N, int P, int H, int H_kv, int d,
    const int32_t* cu_seqlens, int num_seqs,
    int rank_lo, int rank_hi, cudaStream_t stream);

/* Head fragments ("fragmentation by heads": q2bstudio.com, "Ulysses Unleashed:
 * Context Parallelism with Fragmentation by Heads" -- a rank may process its
 * heads a few at a time, one fragment after another, so that only one
 * fragment's full-sequence activations exist at once).
 * ulysses_a2a_seq_to_head_frag gathers global query heads
 * [head_lo, head_lo + num_heads) of every token from the P sequence shards
 * x0_seq ([N/P, H, d] each) into ONE buffer x0_frag [N, num_heads, d], and
 * likewise their key/value heads [head_lo/g, (head_lo + num_heads)/g)
 * (g = H/H_kv) from x1_seq/x2_seq ([N/P, H_kv, d]) into x1_frag/x2_frag
 * [N, num_heads/g, d]; ulysses_a2a_head_to_seq_frag is the exact inverse and
 * writes only the fragment's head columns of the sequence shards.
 * The fragment must be whole GQA groups (head_lo and num_heads multiples of g)
 * inside one rank's heads [r*H/P, (r+1)*H/P); else ULY_ERR_INVALID_ARG.
 * Attention on a fragment is ulysses_attn_fwd / ulysses_attn_bwd with P = 1,
 * H = num_heads, H_kv = num_heads/g on the fragment buffers (heads do not
 * interact). x1/x2 may be NULL (both sides). Bit copies; all pointers 16-byte
 * aligned; caller-owned; asynchronous on `stream`. */
ULY_API uly_status ulysses_a2a_seq_to_head_frag(
    const void* const* x0_seq, const void* const* x1_seq, const void* const* x2_seq,
    void* x0_frag, void* x1_frag, void* x2_frag,
    int64_t N, int P, int H, int H_kv, int d, int head_lo, int num_heads, cudaStream_t stream);
ULY_API uly_status ulysses_a2a_head_to_seq_frag(
    const void* x0_frag, const void* x1_frag, const void* x2_frag,
    void* const* x0_seq, void* const* x1_seq, void* const* x2_seq,
    int64_t N, int P, int H, int H_kv, int d, int head_lo, int num_heads, cudaStream_t stream);

/* Pack / unpack for the exchange between processes (one process per GPU, each
 * holding ONE rank's sequence shards; the all-to-all itself is a collective
 * such as NCCL's). The method's first all-to-all sends, from every rank, each
 * token's slice for every other rank's heads, so that each rank then holds
 * the whole sequence for its own heads; the second undoes it
 * (theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually Work?";
 * the Spanish note on contenidos2-1ml.pages.dev, "¿Qué cambia en la
 * práctica…?", wants NVLink for this exchange).
 * Sizes are those of the whole layer (N tokens in all, P ranks; this rank holds
 * n = N/P). A head chunk [head_lo, head_lo + num_heads) inside every rank's H/P
 * query heads (whole GQA groups: head_lo and num_heads multiples of
 * g = H/H_kv, head_lo + num_heads <= H/P) and its key/value heads
 * [head_lo/g, (head_lo + num_heads)/g) inside every rank's H_kv/P move; the
 * chunk lets the exchange of one chunk overlap the attention of another.
 * ulysses_a2a_pack: x0_seq [n, H, d] (x1_seq, x2_seq [n, H_kv, d]) of this
 *   rank -> x0_send [P][n][f][d] (f = num_heads; f/g for slots 1, 2) with
 *   x0_send[q][s][j] = x0_seq[s][q*H/P + head_lo + j]: chunk q is what rank q
 *   must receive. After an all-to-all that delivers chunk q to rank q (in
 *   source-rank order), each rank's receive buffer IS its [N, f, d] head
 *   fragment (token p*n + s came from rank p), ready for ulysses_attn_fwd /
 *   ulysses_attn_bwd with P = 1, H = f, H_kv = f/g.
 * ulysses_a2a_unpack: the inverse, x0_recv [P][n][f][d] -> the chunk's head
 *   columns of x0_seq (other columns untouched). The attention output [N, f, d]
 *   of a rank is already [P][n][f][d] and is sent as is.
 * x1/x2 may be NULL (both sides). Bit copies; pointers 16-byte aligned;
 * caller-owned; asynchronous on `stream`. ULY_ERR_INVALID_ARG for a bad chunk
 * or pointer, ULY_ERR_UNSUPPORTED beyond H*d <= 16384. */
ULY_API uly_status ulysses_a2a_pack(
    const void* x0_seq, const void* x1_seq, const void* x2_seq,
    void* x0_send, void* x1_send, void* x2_send,
    int64_t N, int P, int H, int H_kv, int d, int head_lo, int num_heads, cudaStream_t stream);
ULY_API uly_status ulysses_a2a_unpack(
    const void* x0_recv, const void* x1_recv, const void* x2_recv,
    void* x0_seq, void* x1_seq, void* x2_seq,
    int64_t N, int P, int H, int H_kv, int d, int head_lo, int num_heads, cudaStream_t stream);

/* The projections on either side of the exchange, with the all-to-alls folded
 * into the GEMMs (each rank projects its own tokens before the first
 * all-to-all and its own shard after the second: theaicatchup.com, "How Does
 * Ulysses Sequence Parallelism Actually Work?").
 * ulysses_qkv_proj_seq_to_head: for every token t of every sequence shard,
 *   [q_t | k_t | v_t] = x_t W_qkv^T  (fp32 accumulation, bf16 round to nearest
 *   even), with x_seq[p] [N/P, hidden], w_qkv [(H + 2 H_kv) d, hidden]
 *   row-major (rows 0..H d-1 give Q heads in order, then K heads, then V
 *   heads), written straight into the head shards q_head/k_head/v_head of all
 *   P ranks ([N, H/P, d] and [N, H_kv/P, d]): the same result as projecting
 *   into sequence shards and calling ulysses_a2a_seq_to_head.
 * ulysses_out_proj_head_to_seq: y_t = o_t W_o^T with o_t gathered from the
 *   head shards o_head (all P ranks) and w_o [hidden, H d], written into the
 *   sequence shards y_seq[p] [N/P, hidden]: the same result as
 *   ulysses_a2a_head_to_seq followed by the projection.
 * Needs (N/P) % 128 == 0, hidden % 256 == 0 and (H + 2 H_kv) d % 256 == 0
 * (else ULY_ERR_UNSUPPORTED); other shape rules as the layer. All pointers
 * 16-byte aligned device memory owned by the caller; asynchronous. */
ULY_API uly_status ulysses_qkv_proj_seq_to_head(
    const void* const* x_seq, const void* w_qkv,
    void* const* q_head, void* const* k_head, void* const* v_head,
    int64_t N, int P, int H, int H_kv, int d, int hidden, cudaStream_t stream);
ULY_API uly_status ulysses_out_proj_head_to_seq(
    const void* const* o_head, const void* w_o, void* const* y_seq,
    int64_t N, int P, int H, int H_kv, int d, int hidden, cudaStream_t stream);

/* Backward of the two projections (the gradient of the formulas above; the
 * pages train through the block but do not write its backward), with the
 * all-to-alls again folded into the GEMMs' loads and stores:
 * ulysses_out_proj_bwd: from dy_seq[p] [N/P, hidden] (gradient of Y),
 *   do_head = dY W_o written straight into the head shards ([N, H/P, d] per
 *   rank: the input of ulysses_attn_bwd, no seq->head permute of dO), and
 *   dw_o = sum over all tokens of dy_t^T o_t  ([hidden, H d]), with O read
 *   from the head shards o_head.
 * ulysses_qkv_proj_bwd: from the attention gradients dq_head, dk_head, dv_head
 *   (head shards, as ulysses_attn_bwd writes them), dx_seq[p] = [dq|dk|dv]_t
 *   W_qkv (sequence shards [N/P, hidden]: no head->seq permute of dQ, dK, dV),
 *   and dw_qkv = sum over all tokens of [dq|dk|dv]_t^T x_t
 *   ([(H + 2 H_kv) d, hidden]).
 * dO and dX: fp32 accumulation over the whole reduction, one bf16 rounding
 * (RNE). dw_o and dw_qkv are fp32 (they sum over every token): the call
 * zeroes them and adds the partial sums of 4096-token chunks into them (fp32
 * additions in L2, so their low bits may differ run to run); they are not
 * accumulated across calls. Shape rules as the forward projections;
 * ulysses_out_proj_bwd also needs H d % 256 == 0. */
ULY_API uly_status ulysses_out_proj_bwd(
    const void* const* o_head, const void* w_o, const void* const* dy_seq,
    void* const* do_head, void* dw_o,
    int64_t N, int P, int H, int H_kv, int d, int hidden, cudaStream_t stream);
ULY_API uly_status ulysses_qkv_proj_bwd(
    const void* const* x_seq, const void* w_qkv,
    const void* const* dq_head, const void* const* dk_head, const void* const* dv_head,
    void* const* dx_seq, void* dw_qkv,
    int64_t N, int P, int H, int H_kv, int d, int hidden, cudaStream_t stream);

/* Causal (optionally packed-varlen) grouped-query flash attention forward on the
 * head shards of ranks [rank_lo, rank_hi): each rank runs attention by itself on
 * its heads, which do not interact (theaicatchup.com, ibid., citing DeepSpeed-Ulysses):
 *   s_ij = softmax_scale * q_i.k_j  for j <= i in the same document,
 *   o_i = sum_j softmax_j(s_i) v_j  (bf16, round to nearest even),
 *   lse_i = ln sum_j exp(s_ij)      (float32, layout [H/P, N]).
 * Inputs q_head (H/P heads), k_head/v_head (H_kv/P heads) per rank; outputs
 * o_head and lse_head per rank. softmax_scale <= 0 selects 1/sqrt(d).
 * causal must be 1 (ULY_ERR_UNSUPPORTED otherwise). max_seqlen is a hint
 * (longest document; <= 0 = unknown). fp32 accumulation and softmax. */
ULY_API uly_status ulysses_attn_fwd(
    const void* const* q_head, const void* const* k_head, const void* const* v_head,
    void* const* o_head, float* const* lse_head,
    int64_t N, int P, int H, int H_kv, int d,
    const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
    float softmax_scale, int causal,
    int rank_lo, int rank_hi, cudaStream_t stream);

/* Fused layer forward: the seq->head all-to-all, ulysses_attn_fwd and the
 * head->seq all-to-all in ONE launch. The kernel fetches each rank's Q/K/V
 * tiles straight from the sequence shards (rank r's heads are a column slice
 * of every shard row) and stores O straight into the sequence shards, so no
 * head-sharded copy is ever written: the exchange happens in the addressing.
 * Results are bit-identical to the three separate calls.
 *   q_seq (H heads), k_seq, v_seq (H_kv heads): all P sequence shards,
 *   o_seq: all P sequence shards (only the head columns of ranks
 *   [rank_lo, rank_hi) are written), lse_head: per rank in range, [H/P, N].
 * Needs (N/P) % 128 == 0 (a 128-token tile never straddles two shards);
 * otherwise ULY_ERR_UNSUPPORTED. Everything else as ulysses_attn_fwd. */
ULY_API uly_status ulysses_attn_fwd_seq(
    const void* const* q_seq, const void* const* k_seq, const void* const* v_seq,
    void* const* o_seq, float* const* lse_head,
    int64_t N, int P, int H, int H_kv, int d,
    const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
    float softmax_scale, int causal,
    int rank_lo, int rank_hi, cudaStream_t stream);

/* Bytes of device workspace ulysses_attn_bwd needs for these sizes and this
 * `deterministic` setting: per (rank, query head, row padded to a multiple of
 * 128) the fp32 values lse_i*log2(e) and D_i = dO_i . O_i, for all P ranks;
 * with deterministic == 0 and d == 128 also an fp32 dQ accumulator of
 * (N padded) * H * d floats. Returns 0 for an invalid shape. */
ULY_API size_t ulysses_attn_bwd_workspace_size(int64_t N, int P, int H, int H_kv, int d, int deterministic);

/* Attention backward on the head shards of ranks [rank_lo, rank_hi). The pages
 * train through the layer but do not write its backward; this is the gradient
 * of the forward above (softmax-attention calculus):
 *   P_ij = exp(s_ij - lse_i), D_i = dO_i . O_i,
 *   dV_j = sum_i P_ij dO_i,   dS_ij = P_ij (dO_i.v_j - D_i),
 *   dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i,
 * with dK/dV summed over the H/H_kv query heads of each group. Inputs: q, k, v,
 * o, do_head (head shards, as in the forward) and lse_head from the forward.
 * Outputs dq_head (H/P heads), dk_head, dv_head (H_kv/P heads), bf16.
 * workspace: caller-owned device memory of at least
 * ulysses_attn_bwd_workspace_size() bytes (same `deterministic`), 256-byte
 * aligned; its contents on entry do not matter.
 * deterministic != 0: two passes (K/V-stationary dK, dV; Q-stationary dQ) that
 * recompute S and dP, no atomics: bit-identical results run to run.
 * deterministic == 0 (d == 128): one pass computes dK, dV and dQ together and
 * sums dQ in fp32 with vector reductions in L2 (about 5/7 of the tensor work);
 * dK and dV are the same bits as the two-pass path, dQ agrees to fp32 rounding
 * but its low bits may differ between runs. With d == 64 both settings run
 * the two-pass kernels, and so does deterministic == 0 on a device where the
 * one-pass kernel's shared-memory layout would not fit (see
 * ulysses_attn_bwd_onepass_layout_fits); that choice is made on the host and
 * never turns into an error status. */
ULY_API uly_status ulysses_attn_bwd(
    const void* const* q_head, const void* const* k_head, const void* const* v_head,
    const void* const* o_head, const float* const* lse_head, const void* const* do_head,
    void* const* dq_head, void* const* dk_head, void* const* dv_head,
    int64_t N, int P, int H, int H_kv, int d,
    const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
    float softmax_scale, int deterministic,
    void* workspace, size_t workspace_bytes,
    int rank_lo, int rank_hi, cudaStream_t stream);

/* Fused layer backward: the seq->head all-to-all of dO, ulysses_attn_bwd and
 * the head->seq all-to-all of dQ, dK, dV, reading Q, K, V, O, dO from the
 * sequence shards and writing dQ, dK, dV into them (all arrays: P sequence
 * shards; lse_head: per rank in range, from ulysses_attn_fwd_seq or
 * ulysses_attn_fwd). Workspace and `deterministic` as ulysses_attn_bwd (at
 * least ulysses_attn_bwd_workspace_size() bytes); given
 * ulysses_attn_bwd_seq_workspace_size() bytes, the one-pass mode first copies
 * Q and dO into head shards inside the workspace (two permute launches) and
 * streams them from there, which is faster than from the sequence shards.
 * Bit-identical to the separate calls either way (for dQ with
 * deterministic == 0: up to the run-to-run order of the fp32 sums). Needs
 * (N/P) % 128 == 0; otherwise ULY_ERR_UNSUPPORTED. */
/* Workspace bytes with which ulysses_attn_bwd_seq stages Q and dO in head
 * shards: ulysses_attn_bwd_workspace_size() plus, in the one-pass mode
 * (deterministic == 0, d == 128), 2 * P * N * (H/P) * d * 2 bytes. 0 if the
 * shape is unsupported. */
ULY_API size_t ulysses_attn_bwd_seq_workspace_size(int64_t N, int P, int H, int H_kv, int d, int deterministic);

ULY_API uly_status ulysses_attn_bwd_seq(
    const void* const* q_seq, const void* const* k_seq, const void* const* v_seq,
    const void* const* o_seq, const float* const* lse_head, const void* const* do_seq,
    void* const* dq_seq, void* const* dk_seq, void* const* dv_seq,
    int64_t N, int P, int H, int H_kv, int d,
    const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
    float softmax_scale, int deterministic,
    void* workspace, size_t workspace_bytes,
    int rank_lo, int rank_hi, cudaStream_t stream);

/* The attention backward for callers that cannot allocate device memory: a
 * plugin or embedded runtime that hands this library only its input and output
 * buffers and owns every allocation itself, or a loop where cudaMalloc (which
 * can synchronise the device) is not allowed. The paper has no counterpart;
 * this is a deployment variant of ulysses_attn_bwd with deterministic = 1 and
 * identical arguments and results, minus deterministic/workspace/workspace_bytes.
 *
 * Its scratch is a fixed 32 MiB device array inside this library (held by every
 * GPU that loads the library until the process exits); it needs
 * ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, 1) <= 32 MiB, i.e.
 * H * (N rounded up to a multiple of 128) <= 4,194,304 (for example
 * N <= 131072 at H = 32); larger sizes return ULY_ERR_UNSUPPORTED with nothing
 * launched. It calls no allocator. The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture. Every call shares the one
 * array and leaves its contents behind; the kernels overwrite all of it that
 * they read, so nothing needs clearing, but calls that overlap on the GPU (on
 * different streams, or from different threads) race on it: serialise them. */
ULY_API uly_status ulysses_attn_bwd_noalloc(
    const void* const* q_head, const void* const* k_head, const void* const* v_head,
    const void* const* o_head, const float* const* lse_head, const void* const* do_head,
    void* const* dq_head, void* const* dk_head, void* const* dv_head,
    int64_t N, int P, int H, int H_kv, int d,
    const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
    float softmax_scale,
    int rank_lo, int rank_hi, cudaStream_t stream);

/* Static text for a status code. */
ULY_API const char* ulysses_status_string(uly_status s);

/* Reads and clears the library's device-side error word on the current device
 * (set by a bounded wait that gave up, or by a kernel's own bounds check).
 * Synchronises `stream`. Returns ULY_OK, ULY_ERR_TIMEOUT or ULY_ERR_CUDA;
 * *detail (may be NULL) receives the raw word (0 = clean). */
ULY_API uly_status ulysses_get_device_status(cudaStream_t stream, uint32_t* detail);

/* Test hook: caps every bounded device-side wait at `iters` polls (0 restores
 * the default). Waits that drain a CTA before it exits always keep the default
 * cap. Synchronous; applies to the current device. */
ULY_API void ulysses_set_wait_limit(uint32_t iters);

/* Host-side selection rule of the backward (no CUDA call): returns 1 if the
 * one-pass kernel's shared-memory layout fits when its dynamic shared memory
 * starts `dyn_smem_offset` bytes into the CTA's shared window (the per-block
 * reserved shared memory plus the kernel's static shared memory), else 0.
 * ulysses_attn_bwd with deterministic = 0 applies this rule to the current
 * device once and runs the two-pass kernels when it returns 0 (same dK/dV
 * bits; dQ equal up to the order of its fp32 sums) instead of failing. */
ULY_API int ulysses_attn_bwd_onepass_layout_fits(uint32_t dyn_smem_offset);

/* Test hook: launches one tiny kernel on `stream` that waits, bounded, on an
 * mbarrier nothing arrives on (the same wait routine the attention kernels use),
 * so the wait runs out and records kernel id 0x7F, site 0xABC in the device
 * error word. Nothing faults, traps or hangs; read the result with
 * ulysses_get_device_status(). Use ulysses_set_wait_limit() first to keep it short. */
ULY_API uly_status ulysses_selftest_bounded_wait(cudaStream_t stream);

/* ---------------------------------------------------------------- host-to-host steps
 * The layer with its inputs and outputs in HOST memory (theaicatchup.com, "How
 * Does Ulysses Sequence Parallelism Actually Work?": sequence shards in,
 * sequence shards out). Each submitted step copies the step's sequence shards
 * Q, K, V (and dO when backward != 0) from host memory to the GPU, runs
 * ulysses_a2a_seq_to_head, ulysses_attn_fwd, ulysses_a2a_head_to_seq of O (and
 * ulysses_a2a_seq_to_head of dO, ulysses_attn_bwd, ulysses_a2a_head_to_seq of
 * dQ, dK, dV), and copies O (and dQ, dK, dV) back to host memory. Results are
 * bit-identical to those calls made one by one.
 *
 * Copies in, compute and copies out run on three streams the handle creates,
 * with two alternating sets of sequence-side device buffers, so the copies of
 * neighbouring steps overlap this step's kernels and PCIe carries both
 * directions at once. The caller owns the device memory: one scratch buffer
 * of ulysses_host_pipeline_scratch_bytes() bytes, 256-byte aligned, that must
 * outlive the handle and is used by nothing else meanwhile. The handle owns
 * only host memory, its streams and its events. A handle is not thread-safe:
 * calls on one handle must not overlap (different handles may be used from
 * different threads). */
typedef struct uly_host_pipeline uly_host_pipeline;

/* Scratch bytes for the shape (0 if the shape is unsupported). Two sets of
 * sequence-side buffers, the head-side buffers, the LSE and, with backward,
 * the ulysses_attn_bwd workspace of the given mode. */
ULY_API size_t ulysses_host_pipeline_scratch_bytes(int64_t N, int P, int H, int H_kv, int d, int backward,
                                                   int deterministic);

/* Creates a handle over `scratch` (device, 256-byte aligned, scratch_bytes at
 * least the size above). *out is NULL on failure. Status: ULY_ERR_INVALID_ARG
 * (NULL out or scratch, misaligned or short scratch), ULY_ERR_UNSUPPORTED
 * (shape), ULY_ERR_CUDA (stream or event creation). */
ULY_API uly_status ulysses_host_pipeline_create(int64_t N, int P, int H, int H_kv, int d, int backward,
                                                int deterministic, void* scratch, size_t scratch_bytes,
                                                uly_host_pipeline** out);

/* Enqueues one step and returns without waiting. *_host: HOST arrays of P
 * HOST pointers, one sequence shard each ([N/P, Hx, d] bf16, 16-byte aligned;
 * pinned memory for the copies to be asynchronous). dO, dQ, dK, dV are read
 * only with backward (may be NULL otherwise). The input shards must stay
 * unchanged and the output shards unread until the step's copies are done:
 * after `after` (if not NULL) has completed, or after
 * ulysses_host_pipeline_synchronize(). cu_seqlens as everywhere (DEVICE
 * array, or NULL); softmax_scale 0 = 1/sqrt(d). before / after: caller-owned
 * CUDA events (or NULL) recorded on the copy-in stream before the step's first
 * copy and on the copy-out stream after its last. Validation failures return
 * before anything is enqueued; a launch failure returns ULY_ERR_CUDA. */
ULY_API uly_status ulysses_host_pipeline_submit(uly_host_pipeline* pipe, const void* const* q_host,
                                                const void* const* k_host, const void* const* v_host,
                                                const void* const* do_host, void* const* o_host,
                                                void* const* dq_host, void* const* dk_host, void* const* dv_host,
                                                const int32_t* cu_seqlens, int num_seqs, float softmax_scale,
                                                cudaEvent_t before, cudaEvent_t after);

/* Waits for every step submitted so far. */
ULY_API uly_status ulysses_host_pipeline_synchronize(uly_host_pipeline* pipe);

/* Waits for the submitted steps, then releases the handle's streams, events
 * and host memory (not the scratch buffer). NULL is accepted. */
ULY_API uly_status ulysses_host_pipeline_destroy(uly_host_pipeline* pipe);

#ifdef __cplusplus
}
#endif
#endif /* ULYSSES_B200_H */
