// Host-to-host layer steps: the step's sequence shards are copied from host
// memory, the layer runs (all-to-all #1, attention, all-to-all #2, and the
// backward), and the results are copied back, with the copies of neighbouring
// steps overlapping this step's kernels. The pages' layer takes sequence shards
// and returns sequence shards (theaicatchup.com, "How Does Ulysses Sequence
// Parallelism Actually Work?"); this is that layer with its inputs and outputs
// in host memory.
//
// Three streams: copies in, compute, copies out. Two sets of sequence-side
// device buffers alternate between steps; the head-side buffers, the LSE and
// the backward workspace are shared (the compute stream runs one step at a
// time). Events order the streams:
//   copy-in  (step k, set j) waits for compute (step k-2) to finish with set j
//   compute  (step k)        waits for copy-in (step k) and for copy-out
//                             (step k-2) to finish reading set j's outputs
//   copy-out (step k)        waits for compute (step k)
// All device memory is the caller's scratch buffer; the handle holds only the
// streams, the events and the carved-up pointers.

#include <new>

namespace {

constexpr int kIn = 4, kOut = 4;   // q, k, v, dO  /  o, dQ, dK, dV

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Carves the scratch buffer (or, with base == nullptr, only measures it).
struct ScratchPlan {
  size_t bytes = 0;
  char* base = nullptr;
  void* take(size_t n) {
    void* p = base ? base + bytes : nullptr;
    bytes += align_up(n);
    return p;
  }
};

}  // namespace

struct uly_host_pipeline {
  int64_t N;
  int P, H, H_kv, d, backward, deterministic;
  cudaStream_t s_in, s_comp, s_out;
  cudaEvent_t loaded[2], computed[2], out_done[2];
  uint64_t step;
  void* in[2][kIn][ULY_MAX_RANKS];
  void* out[2][kOut][ULY_MAX_RANKS];
  void* head[kIn + kOut][ULY_MAX_RANKS];   // q, k, v, dO, o, dQ, dK, dV head shards
  float* lse[ULY_MAX_RANKS];
  void* ws;
  size_t ws_bytes;
  size_t shard_bytes[2];                  // [0]: H heads, [1]: H_kv heads (sequence and head shards alike)
};

namespace {

// Heads of tensor t in either list: q, o, dO, dQ have H; k, v, dK, dV have H_kv.
int is_kv(int t) { return t == 1 || t == 2; }

size_t plan_scratch(ScratchPlan& sp, uly_host_pipeline* hp, int64_t N, int P, int H, int H_kv, int d, int backward,
                    int deterministic) {
  const size_t sb[2] = {static_cast<size_t>(N / P) * H * d * 2, static_cast<size_t>(N / P) * H_kv * d * 2};
  const int nt = backward ? 4 : 3, no = backward ? 4 : 1;
  for (int j = 0; j < 2; ++j) {
    for (int t = 0; t < nt; ++t)
      for (int p = 0; p < P; ++p) {
        void* q = sp.take(sb[is_kv(t)]);
        if (hp) hp->in[j][t][p] = q;
      }
    for (int t = 0; t < no; ++t)
      for (int p = 0; p < P; ++p) {
        void* q = sp.take(sb[t >= 2 ? 1 : 0]);
        if (hp) hp->out[j][t][p] = q;
      }
  }
  for (int t = 0; t < kIn + kOut; ++t) {
    const bool used = t < 3 || t == 4 || (backward && (t == 3 || t >= 5));
    if (!used) continue;
    const bool kv = t == 1 || t == 2 || t == 6 || t == 7;
    for (int p = 0; p < P; ++p) {
      void* q = sp.take(sb[kv ? 1 : 0]);
      if (hp) hp->head[t][p] = q;
    }
  }
  for (int p = 0; p < P; ++p) {
    void* q = sp.take(static_cast<size_t>(H / P) * N * sizeof(float));
    if (hp) hp->lse[p] = static_cast<float*>(q);
  }
  const size_t ws = backward ? ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, deterministic) : 0;
  void* w = ws ? sp.take(ws) : nullptr;
  if (hp) {
    hp->ws = w;
    hp->ws_bytes = ws;
    hp->shard_bytes[0] = sb[0];
    hp->shard_bytes[1] = sb[1];
  }
  return sp.bytes;
}

}  // namespace

extern "C" {

size_t ulysses_host_pipeline_scratch_bytes(int64_t N, int P, int H, int H_kv, int d, int backward,
                                           int deterministic) {
  if (check_shape(N, P, H, H_kv, d, 0, P > 0 ? P : 1) != ULY_OK) return 0;
  ScratchPlan sp;
  return plan_scratch(sp, nullptr, N, P, H, H_kv, d, backward ? 1 : 0, deterministic ? 1 : 0);
}

uly_status ulysses_host_pipeline_create(int64_t N, int P, int H, int H_kv, int d, int backward, int deterministic,
                                        void* scratch, size_t scratch_bytes, uly_host_pipeline** out) {
  if (out == nullptr) return ULY_ERR_INVALID_ARG;
  *out = nullptr;
  uly_status st = check_shape(N, P, H, H_kv, d, 0, P);
  if (st != ULY_OK) return st;
  backward = backward ? 1 : 0;
  deterministic = deterministic ? 1 : 0;
  if (scratch == nullptr || (reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return ULY_ERR_INVALID_ARG;
  if (scratch_bytes < ulysses_host_pipeline_scratch_bytes(N, P, H, H_kv, d, backward, deterministic))
    return ULY_ERR_INVALID_ARG;
  uly_host_pipeline* hp = new (std::nothrow) uly_host_pipeline;
  if (hp == nullptr) return ULY_ERR_INVALID_ARG;
  memset(hp, 0, sizeof(*hp));
  hp->N = N;
  hp->P = P;
  hp->H = H;
  hp->H_kv = H_kv;
  hp->d = d;
  hp->backward = backward;
  hp->deterministic = deterministic;
  ScratchPlan sp;
  sp.base = static_cast<char*>(scratch);
  plan_scratch(sp, hp, N, P, H, H_kv, d, backward, deterministic);
  bool ok = cudaStreamCreateWithFlags(&hp->s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp->s_out, cudaStreamNonBlocking) == cudaSuccess;
  for (int j = 0; j < 2 && ok; ++j)
    ok = cudaEventCreateWithFlags(&hp->loaded[j], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp->computed[j], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp->out_done[j], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    ulysses_host_pipeline_destroy(hp);
    return ULY_ERR_CUDA;
  }
  *out = hp;
  return ULY_OK;
}

uly_status ulysses_host_pipeline_submit(uly_host_pipeline* hp, const void* const* q_host, const void* const* k_host,
                                        const void* const* v_host, const void* const* do_host, void* const* o_host,
                                        void* const* dq_host, void* const* dk_host, void* const* dv_host,
                                        const int32_t* cu_seqlens, int num_seqs, float softmax_scale,
                                        cudaEvent_t before, cudaEvent_t after) {
  if (hp == nullptr) return ULY_ERR_INVALID_ARG;
  const int P = hp->P;
  const void* const* hin[kIn] = {q_host, k_host, v_host, do_host};
  void* const* hout[kOut] = {o_host, dq_host, dk_host, dv_host};
  const int nt = hp->backward ? 4 : 3, no = hp->backward ? 4 : 1;
  for (int t = 0; t < nt; ++t)
    if (!ranks_ok(hin[t], 0, P)) return ULY_ERR_INVALID_ARG;
  for (int t = 0; t < no; ++t)
    if (!ranks_ok(reinterpret_cast<const void* const*>(hout[t]), 0, P)) return ULY_ERR_INVALID_ARG;
  if (check_cu(cu_seqlens, num_seqs, hp->N) != ULY_OK) return ULY_ERR_INVALID_ARG;
  const int j = static_cast<int>(hp->step & 1u);
  const int64_t N = hp->N;
  const int H = hp->H, Hk = hp->H_kv, d = hp->d;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t x) { if (e == cudaSuccess) e = x; return e == cudaSuccess; };
  auto okst = [&](uly_status s) { if (s != ULY_OK && e == cudaSuccess) e = cudaErrorLaunchFailure; return s; };
  // copies in: one cudaMemcpyAsync per shard
  if (before != nullptr) ok(cudaEventRecord(before, hp->s_in));
  ok(cudaStreamWaitEvent(hp->s_in, hp->computed[j], 0));
  for (int t = 0; t < nt && e == cudaSuccess; ++t)
    for (int p = 0; p < P; ++p)
      ok(cudaMemcpyAsync(hp->in[j][t][p], hin[t][p], hp->shard_bytes[is_kv(t)], cudaMemcpyHostToDevice, hp->s_in));
  ok(cudaEventRecord(hp->loaded[j], hp->s_in));
  // the layer
  ok(cudaStreamWaitEvent(hp->s_comp, hp->loaded[j], 0));
  ok(cudaStreamWaitEvent(hp->s_comp, hp->out_done[j], 0));
  uly_status st = ULY_OK;
  auto head = [&](int t) { return static_cast<void* const*>(hp->head[t]); };
  auto chead = [&](int t) { return static_cast<const void* const*>(hp->head[t]); };
  auto in = [&](int t) { return static_cast<const void* const*>(hp->in[j][t]); };
  auto outp = [&](int t) { return static_cast<void* const*>(hp->out[j][t]); };
  if (e == cudaSuccess) {
    st = okst(ulysses_a2a_seq_to_head(in(0), in(1), in(2), head(0), head(1), head(2), N, P, H, Hk, d, cu_seqlens,
                                      num_seqs, 0, P, hp->s_comp));
    if (st == ULY_OK)
      st = okst(ulysses_attn_fwd(chead(0), chead(1), chead(2), head(4), hp->lse, N, P, H, Hk, d, cu_seqlens,
                                 num_seqs, 0, softmax_scale, 1, 0, P, hp->s_comp));
    if (st == ULY_OK)
      st = okst(ulysses_a2a_head_to_seq(chead(4), nullptr, nullptr, outp(0), nullptr, nullptr, N, P, H, Hk, d,
                                        cu_seqlens, num_seqs, 0, P, hp->s_comp));
    if (st == ULY_OK && hp->backward) {
      st = okst(ulysses_a2a_seq_to_head(in(3), nullptr, nullptr, head(3), nullptr, nullptr, N, P, H, Hk, d,
                                        cu_seqlens, num_seqs, 0, P, hp->s_comp));
      if (st == ULY_OK)
        st = okst(ulysses_attn_bwd(chead(0), chead(1), chead(2), chead(4),
                                   static_cast<const float* const*>(hp->lse), chead(3), head(5), head(6), head(7), N,
                                   P, H, Hk, d, cu_seqlens, num_seqs, 0, softmax_scale, hp->deterministic, hp->ws,
                                   hp->ws_bytes, 0, P, hp->s_comp));
      if (st == ULY_OK)
        st = okst(ulysses_a2a_head_to_seq(chead(5), chead(6), chead(7), outp(1), outp(2), outp(3), N, P, H, Hk, d,
                                          cu_seqlens, num_seqs, 0, P, hp->s_comp));
    }
  }
  ok(cudaEventRecord(hp->computed[j], hp->s_comp));
  // copies out
  ok(cudaStreamWaitEvent(hp->s_out, hp->computed[j], 0));
  for (int t = 0; t < no && e == cudaSuccess; ++t)
    for (int p = 0; p < P; ++p)
      ok(cudaMemcpyAsync(hout[t][p], hp->out[j][t][p], hp->shard_bytes[t >= 2 ? 1 : 0], cudaMemcpyDeviceToHost,
                         hp->s_out));
  ok(cudaEventRecord(hp->out_done[j], hp->s_out));
  if (after != nullptr) ok(cudaEventRecord(after, hp->s_out));
  hp->step += 1;
  if (st != ULY_OK) return st;
  return from_cuda(e);
}

uly_status ulysses_host_pipeline_synchronize(uly_host_pipeline* hp) {
  if (hp == nullptr) return ULY_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(hp->s_in);
  cudaError_t e2 = cudaStreamSynchronize(hp->s_comp);
  cudaError_t e3 = cudaStreamSynchronize(hp->s_out);
  return from_cuda(e != cudaSuccess ? e : (e2 != cudaSuccess ? e2 : e3));
}

uly_status ulysses_host_pipeline_destroy(uly_host_pipeline* hp) {
  if (hp == nullptr) return ULY_OK;
  cudaStream_t ss[3] = {hp->s_in, hp->s_comp, hp->s_out};
  for (cudaStream_t s : ss)
    if (s != nullptr) cudaStreamSynchronize(s);
  for (int j = 0; j < 2; ++j) {
    if (hp->loaded[j]) cudaEventDestroy(hp->loaded[j]);
    if (hp->computed[j]) cudaEventDestroy(hp->computed[j]);
    if (hp->out_done[j]) cudaEventDestroy(hp->out_done[j]);
  }
  for (cudaStream_t s : ss)
    if (s != nullptr) cudaStreamDestroy(s);
  delete hp;
  return ULY_OK;
}

}  // extern "C"
