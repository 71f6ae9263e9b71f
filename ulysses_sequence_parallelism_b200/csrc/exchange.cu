// Pack and unpack of one rank's sequence shard for the real multi-process
// Ulysses exchange (one process per GPU, the all-to-all itself done by NCCL).
//
// The method's first all-to-all sends, from every rank, the slice of each of
// its tokens that belongs to each other rank's heads, so that every rank ends
// up with the whole sequence for its own heads; the second one undoes it
// (theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually Work?";
// the Spanish note on contenidos2-1ml.pages.dev asks for NVLink so that this
// exchange does not become the bottleneck, "¿Qué cambia en la práctica…?").
//
// Rank p holds the sequence shard x[s, h, :] (s < n = N/P, h < Hx). For a head
// chunk [lo, lo + f) inside every rank's Hx/P heads:
//   pack   : send[q][s, j, :] = x[s, q*(Hx/P) + lo + j, :]      (q < P, j < f)
//   unpack : x[s, q*(Hx/P) + lo + j, :] = recv[q][s, j, :]
// send/recv are [P][n][f][d]. An all-to-all that delivers send chunk q to rank
// q turns rank q's receive buffer, source rank by source rank, into
// [N, f, d]: the whole sequence of its f heads (token p*n + s from rank p),
// the head-side layout the attention kernels read. On the way back the
// attention output [N, f, d] is already [P][n][f][d] and is sent as is; the
// receiving rank unpacks it. With lo = 0 and f = Hx/P the chunk is all heads.
//
// HBM-bound copy: every byte read once and written once; 16-byte vectors;
// each thread owns fixed columns of a row so the index arithmetic is hoisted;
// runs of f*d*2 contiguous bytes on the chunk side. Up to three tensors (Q, K,
// V or dQ, dK, dV) in one launch.
#include "common.cuh"
#include "kernels.h"

namespace uly {
namespace exchange_impl {

constexpr int kThreads = 256;
constexpr int kMaxVecPerThread = 8;     // P * f * d / 8 <= 2048 vectors moved per row
constexpr int kUnroll = 8;
constexpr int kTargetBlocks = 148 * 8;

struct Slot {
  const void* src;
  void* dst;
  int row_vecs;    // vectors per sequence-side row (Hx * d / 8)
  int hl_vecs;     // vectors per rank's head slice (Hx/P * d / 8)
  int lo_vecs;     // chunk offset inside a rank's slice (lo * d / 8)
  int f_vecs;      // vectors per chunk row (f * d / 8)
};

struct Args {
  Slot slot[3];
  int slot_of[3];
  int n;           // tokens of this rank
  int P;
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

template <bool kPack>
__global__ void __launch_bounds__(kThreads) exchange_kernel(const __grid_constant__ Args a) {
  const Slot& sl = a.slot[a.slot_of[blockIdx.y]];
  const int rv = a.P * sl.f_vecs;                 // vectors moved per sequence-side row
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
  // Per column: offset in the sequence-side row, and in the chunk side
  // (destination rank q's chunk base + offset within a chunk row).
  int seq_off[kMaxVecPerThread];
  int64_t chunk_base[kMaxVecPerThread];
  int chunk_off[kMaxVecPerThread];
  const int64_t chunk_elems = static_cast<int64_t>(a.n) * sl.f_vecs;   // vectors per rank chunk
#pragma unroll
  for (int k = 0; k < kMaxVecPerThread; ++k) {
    const int v = (rv <= kThreads) ? (threadIdx.x - r_off * rv) : (threadIdx.x + k * kThreads);
    const bool ok = k < vpt && v < rv;
    const int q = v / sl.f_vecs;
    const int rem = v - q * sl.f_vecs;
    seq_off[k] = ok ? q * sl.hl_vecs + sl.lo_vecs + rem : -1;
    chunk_base[k] = q * chunk_elems;
    chunk_off[k] = rem;
  }
  const int s_begin = blockIdx.x * a.rows_per_block;
  const int s_end = min(s_begin + a.rows_per_block, a.n);
  const uint4* src = reinterpret_cast<const uint4*>(sl.src);
  uint4* dst = reinterpret_cast<uint4*>(sl.dst);
#pragma unroll 1
  for (int k = 0; k < kMaxVecPerThread; ++k) {
    if (seq_off[k] < 0) continue;
    // sequence side: row s at s*row_vecs + seq_off; chunk side: chunk_base + s*f_vecs + chunk_off
    const int64_t so = seq_off[k], co = chunk_base[k] + chunk_off[k];
    int s = s_begin + r_off;
#pragma unroll 1
    for (; s + (kUnroll - 1) * rows_per_pass < s_end; s += kUnroll * rows_per_pass) {
      uint4 buf[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t su = s + u * rows_per_pass;
        buf[u] = kPack ? ld_stream(src + su * sl.row_vecs + so) : ld_stream(src + co + su * sl.f_vecs);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t su = s + u * rows_per_pass;
        if (kPack) st_vec(dst + co + su * sl.f_vecs, buf[u]);
        else st_vec(dst + su * sl.row_vecs + so, buf[u]);
      }
    }
    for (; s < s_end; s += rows_per_pass) {
      const int64_t su = s;
      if (kPack) st_vec(dst + co + su * sl.f_vecs, ld_stream(src + su * sl.row_vecs + so));
      else st_vec(dst + su * sl.row_vecs + so, ld_stream(src + co + su * sl.f_vecs));
    }
  }
}

}  // namespace exchange_impl

int exchange_max_row_vecs() {
  using namespace exchange_impl;
  return kThreads * kMaxVecPerThread;
}

cudaError_t launch_exchange(bool pack, const void* const src[3], void* const dst[3], const int hx[3],
                            const int lo[3], const int f[3], int64_t N, int P, int d, cudaStream_t stream) {
  using namespace exchange_impl;
  Args a;
  memset(&a, 0, sizeof(a));
  a.n = static_cast<int>(N / P);
  a.P = P;
  const int dvec = d / 8;
  int n_active = 0, max_rpp = 1;
  for (int s = 0; s < 3; ++s) {
    if (src[s] == nullptr || dst[s] == nullptr) continue;
    Slot& sl = a.slot[s];
    sl.src = src[s];
    sl.dst = dst[s];
    sl.row_vecs = hx[s] * dvec;
    sl.hl_vecs = hx[s] / P * dvec;
    sl.lo_vecs = lo[s] * dvec;
    sl.f_vecs = f[s] * dvec;
    a.slot_of[n_active++] = s;
    const int rv = P * sl.f_vecs;
    const int rpp = rv <= kThreads ? kThreads / rv : 1;
    if (rpp > max_rpp) max_rpp = rpp;
  }
  if (n_active == 0 || a.n == 0) return cudaSuccess;
  const int per_slot_blocks = (kTargetBlocks + n_active - 1) / n_active;
  int rpb = (a.n + per_slot_blocks - 1) / per_slot_blocks;
  const int unit = max_rpp * kUnroll;
  rpb = (rpb + unit - 1) / unit * unit;
  a.rows_per_block = rpb;
  dim3 grid((a.n + rpb - 1) / rpb, n_active);
  if (pack)
    exchange_kernel<true><<<grid, kThreads, 0, stream>>>(a);
  else
    exchange_kernel<false><<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace uly
