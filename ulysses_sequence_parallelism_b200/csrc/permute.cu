// Ulysses all-to-all emulation on one GPU: sequence <-> head sharding permutes.
//
// The method's two all-to-alls per layer (theaicatchup.com, "How Does Ulysses
// Sequence Parallelism Actually Work?": the first gives each rank the whole
// sequence for its subset of heads, the second undoes it after attention)
// become, with the P ranks as P buffers of one GPU, pure index maps:
//   seq -> head : head[q][t, j, :] = seq[t / n][t % n, q*Hl + j, :]   (n = N/P, Hl = Hx/P)
//   head -> seq : the inverse.
// HBM-bound: every byte is read once and written once. The kernel walks the
// sequence-side rows (one token of one rank: Hx*d contiguous bf16), so the
// sequence side is streamed contiguously and the head side is written/read in
// contiguous runs of Hl*d*2 bytes (512 B .. 2 KB at the Llama shapes). Each
// thread owns fixed 16-byte columns of a row, so all index arithmetic except
// one multiply-add per row is hoisted out of the copy loop; four rows are in
// flight per thread (ILP) to cover HBM latency.
#include "common.cuh"
#include "kernels.h"

namespace uly {

namespace permute_impl {

constexpr int kThreads = 512;
constexpr int kMaxVecPerThread = 8;     // supports Hx*d/8 <= 4096 vectors per row
constexpr int kUnroll = 8;
constexpr int kTargetBlocks = 148 * 8;  // ~2 waves of 4 resident 512-thread blocks per SM

struct SlotArgs {
  RankPtrs src;
  RankPtrsMut dst;
  int hx;          // heads of this tensor (H or H_kv)
  int active;
};

struct PermuteArgs {
  SlotArgs slot[3];
  int slot_of[3];  // blockIdx.y / P -> slot (active slots only)
  int n;           // tokens per rank (N/P)
  int P;
  int dvec;        // d / 8 : 16-byte vectors per head row
  int rank_lo, rank_hi;
  int rows_per_block;
};

ULY_DEV uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
ULY_DEV void st_vec(uint4* p, const uint4& v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

template <bool kSeqToHead>
__global__ void __launch_bounds__(kThreads) permute_kernel(const __grid_constant__ PermuteArgs a) {
  const int yi = blockIdx.y / a.P;
  const int p = blockIdx.y - yi * a.P;               // sequence-side rank
  const SlotArgs& sl = a.slot[a.slot_of[yi]];
  const int Hl = sl.hx / a.P;
  const int row_vecs = sl.hx * a.dvec;                // vectors per sequence-side row
  const int head_row_vecs = Hl * a.dvec;              // vectors per head-side token row
  const int lo_v = a.rank_lo * head_row_vecs;
  const int rv = (a.rank_hi - a.rank_lo) * head_row_vecs;

  // Column assignment: rows_per_pass rows per pass, vpt vectors per thread per row.
  int rows_per_pass, vpt, r_off;
  if (rv <= kThreads) {
    rows_per_pass = kThreads / rv;
    vpt = 1;
    r_off = threadIdx.x / rv;
    if (r_off >= rows_per_pass) return;
  } else {
    rows_per_pass = 1;
    vpt = (rv + kThreads - 1) / kThreads;
    r_off = 0;
  }
  // Per-column constants: sequence-side offset within the row, head rank, head-side offset.
  int seq_off[kMaxVecPerThread];
  int q_of[kMaxVecPerThread];
  int head_off[kMaxVecPerThread];
#pragma unroll
  for (int k = 0; k < kMaxVecPerThread; ++k) {
    int v = (rv <= kThreads) ? (threadIdx.x - r_off * rv) : (threadIdx.x + k * kThreads);
    bool ok = k < vpt && v < rv;
    int vv = lo_v + v;
    int hx = vv / a.dvec;
    int c = vv - hx * a.dvec;
    int q = hx / Hl;
    int j = hx - q * Hl;
    seq_off[k] = ok ? vv : -1;
    q_of[k] = q;
    head_off[k] = j * a.dvec + c;
  }

  const int s_begin = blockIdx.x * a.rows_per_block;
  int s_end = s_begin + a.rows_per_block;
  if (s_end > a.n) s_end = a.n;
  const uint4* seq_base_c = reinterpret_cast<const uint4*>(sl.src.p[p]);
  uint4* seq_base_m = reinterpret_cast<uint4*>(sl.dst.p[p]);

#pragma unroll 1
  for (int k = 0; k < kMaxVecPerThread; ++k) {
    if (seq_off[k] < 0) continue;
    const int q = q_of[k];
    const uint4* hsrc = kSeqToHead ? nullptr : reinterpret_cast<const uint4*>(sl.src.p[q]);
    uint4* hdst = kSeqToHead ? reinterpret_cast<uint4*>(sl.dst.p[q]) : nullptr;
    int s = s_begin + r_off;
#pragma unroll 1
    for (; s + (kUnroll - 1) * rows_per_pass < s_end; s += kUnroll * rows_per_pass) {
      uint4 buf[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int su = s + u * rows_per_pass;
        const int64_t t = static_cast<int64_t>(p) * a.n + su;
        if (kSeqToHead)
          buf[u] = ld_stream(seq_base_c + static_cast<int64_t>(su) * row_vecs + seq_off[k]);
        else
          buf[u] = ld_stream(hsrc + t * head_row_vecs + head_off[k]);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int su = s + u * rows_per_pass;
        const int64_t t = static_cast<int64_t>(p) * a.n + su;
        if (kSeqToHead)
          st_vec(hdst + t * head_row_vecs + head_off[k], buf[u]);
        else
          st_vec(seq_base_m + static_cast<int64_t>(su) * row_vecs + seq_off[k], buf[u]);
      }
    }
    for (; s < s_end; s += rows_per_pass) {
      const int64_t t = static_cast<int64_t>(p) * a.n + s;
      if (kSeqToHead)
        st_vec(hdst + t * head_row_vecs + head_off[k],
               ld_stream(seq_base_c + static_cast<int64_t>(s) * row_vecs + seq_off[k]));
      else
        st_vec(seq_base_m + static_cast<int64_t>(s) * row_vecs + seq_off[k],
               ld_stream(hsrc + t * head_row_vecs + head_off[k]));
    }
  }
}

}  // namespace permute_impl

int permute_max_row_vecs() {
  using namespace permute_impl; return kThreads * kMaxVecPerThread; }

cudaError_t launch_permute(bool seq_to_head, const void* const* src[3], void* const* dst[3], const int hx[3],
                           int64_t N, int P, int d, int rank_lo, int rank_hi, cudaStream_t stream) {
  using namespace permute_impl;
  PermuteArgs a;
  memset(&a, 0, sizeof(a));
  a.n = static_cast<int>(N / P);
  a.P = P;
  a.dvec = d / 8;
  a.rank_lo = rank_lo;
  a.rank_hi = rank_hi;
  int max_rows_per_pass = 1;
  int n_active = 0;
  for (int s = 0; s < 3; ++s) {
    a.slot[s].active = (src[s] != nullptr && dst[s] != nullptr) ? 1 : 0;
    a.slot[s].hx = hx[s];
    if (!a.slot[s].active) continue;
    a.slot_of[n_active++] = s;
    const bool sr = seq_to_head;
    for (int r = 0; r < P; ++r) {
      // sequence-side buffers: every rank; head-side buffers: ranks in range only.
      bool need_src = sr ? true : (r >= rank_lo && r < rank_hi);
      bool need_dst = sr ? (r >= rank_lo && r < rank_hi) : true;
      a.slot[s].src.p[r] = need_src ? src[s][r] : nullptr;
      a.slot[s].dst.p[r] = need_dst ? dst[s][r] : nullptr;
    }
    int rv = (rank_hi - rank_lo) * (hx[s] / P) * (d / 8);
    int rpp = rv <= kThreads ? kThreads / rv : 1;
    if (rpp > max_rows_per_pass) max_rows_per_pass = rpp;
  }
  if (n_active == 0 || a.n == 0) return cudaSuccess;
  // Rows per block: enough blocks for ~2 waves, each at least one unrolled pass.
  const int per_rank_blocks = (kTargetBlocks + n_active * P - 1) / (n_active * P);
  int rpb = (a.n + per_rank_blocks - 1) / per_rank_blocks;
  const int unit = max_rows_per_pass * kUnroll;
  rpb = (rpb + unit - 1) / unit * unit;
  a.rows_per_block = rpb;
  dim3 grid((a.n + rpb - 1) / rpb, n_active * P);
  if (seq_to_head)
    permute_kernel<true><<<grid, kThreads, 0, stream>>>(a);
  else
    permute_kernel<false><<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace uly
