// Ulysses all-to-all emulation on one GPU: sequence <-> head sharding permutes.
//
// The method's two all-to-alls per layer (theaicatchup.com, "How Does Ulysses
// Sequence Parallelism Actually Work?": the first gives each rank the whole
// sequence for its subset of heads, the second undoes it after attention)
// become, with the P ranks as P buffers of one GPU, pure index maps:
//   seq -> head : head[q][t, j, :] = seq[t / n][t % n, q*Hl + j, :]   (n = N/P, Hl = Hx/P)
//   head -> seq : the inverse.
// The same kernel moves a head fragment of one rank (a whole number of GQA
// groups, processed one after another to shrink activation memory:
// q2bstudio.com, "Ulysses Unleashed", fragmentation by heads): then the head
// side is one buffer [N, f, d] holding global heads [h_lo, h_lo + f).
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
  int hx;          // heads of this tensor on the sequence side (H or H_kv)
  int hb;          // heads per head-side buffer (Hx/P, or the fragment size)
  int h_lo, h_cnt; // global heads moved: [h_lo, h_lo + h_cnt)
  int h_base;      // head-side buffer b holds global heads [h_base + b*hb, +hb)
  int active;
};

struct PermuteArgs {
  SlotArgs slot[3];
  int slot_of[3];  // blockIdx.y / P -> slot (active slots only)
  int n;           // tokens per rank (N/P)
  int P;
  int dvec;        // d / 8 : 16-byte vectors per head row
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
  const int Hl = sl.hb;
  const int row_vecs = sl.hx * a.dvec;                // vectors per sequence-side row
  const int head_row_vecs = Hl * a.dvec;              // vectors per head-side token row
  const int lo_v = sl.h_lo * a.dvec;
  const int rv = sl.h_cnt * a.dvec;

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
    int q = (hx - sl.h_base) / Hl;
    int j = hx - sl.h_base - q * Hl;
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

namespace permute_impl {
// hb/h_lo/h_cnt/h_base per slot as in SlotArgs; nb = head-side buffers used
// (indices [b_lo, b_lo + nb) of the head-side pointer arrays).
cudaError_t launch(bool seq_to_head, const void* const* src[3], void* const* dst[3], const int hx[3],
                   const int hb[3], const int h_lo[3], const int h_cnt[3], const int h_base[3], int b_lo, int nb,
                   int64_t N, int P, int d, cudaStream_t stream) {
  PermuteArgs a;
  memset(&a, 0, sizeof(a));
  a.n = static_cast<int>(N / P);
  a.P = P;
  a.dvec = d / 8;
  int max_rows_per_pass = 1;
  int n_active = 0;
  for (int s = 0; s < 3; ++s) {
    SlotArgs& sl = a.slot[s];
    sl.active = (src[s] != nullptr && dst[s] != nullptr) ? 1 : 0;
    sl.hx = hx[s];
    sl.hb = hb[s];
    sl.h_lo = h_lo[s];
    sl.h_cnt = h_cnt[s];
    sl.h_base = h_base[s];
    if (!sl.active) continue;
    a.slot_of[n_active++] = s;
    const void* const* seq_side = seq_to_head ? src[s] : dst[s];
    const void* const* head_side = seq_to_head ? dst[s] : src[s];
    for (int r = 0; r < P; ++r) {
      if (seq_to_head) sl.src.p[r] = seq_side[r];
      else sl.dst.p[r] = const_cast<void*>(seq_side[r]);
    }
    for (int b = b_lo; b < b_lo + nb; ++b) {      // head-side buffers in use only
      if (seq_to_head) sl.dst.p[b] = const_cast<void*>(head_side[b]);
      else sl.src.p[b] = head_side[b];
    }
    int rv = h_cnt[s] * (d / 8);
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
}  // namespace permute_impl

cudaError_t launch_permute(bool seq_to_head, const void* const* src[3], void* const* dst[3], const int hx[3],
                           int64_t N, int P, int d, int rank_lo, int rank_hi, cudaStream_t stream) {
  int hb[3], h_lo[3], h_cnt[3], h_base[3] = {0, 0, 0};
  for (int s = 0; s < 3; ++s) {
    hb[s] = hx[s] / P;
    h_lo[s] = rank_lo * hb[s];
    h_cnt[s] = (rank_hi - rank_lo) * hb[s];
  }
  return permute_impl::launch(seq_to_head, src, dst, hx, hb, h_lo, h_cnt, h_base, rank_lo, rank_hi - rank_lo, N, P,
                              d, stream);
}

cudaError_t launch_permute_fragment(bool seq_to_head, const void* const* src[3], void* const* dst[3],
                                    const int hx[3], const int f_lo[3], const int f_cnt[3], int64_t N, int P, int d,
                                    cudaStream_t stream) {
  int h_base[3];
  for (int s = 0; s < 3; ++s) h_base[s] = f_lo[s];
  return permute_impl::launch(seq_to_head, src, dst, hx, f_cnt, f_lo, f_cnt, h_base, 0, 1, N, P, d, stream);
}

}  // namespace uly
