// Causal GQA (packed-varlen) flash-attention backward, warp-level mma.sync path.
//
// Gradient of the forward (the pages train through the layer but do not write
// the backward; this is softmax-attention calculus):
//   P_ij = exp(s_ij - lse_i),  D_i = dO_i . O_i
//   dV_j = sum_i P_ij dO_i,   dS_ij = P_ij (dO_i.v_j - D_i)
//   dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
// Three launches: (1) D_i per row and a zeroed fp32 dQ accumulator,
// (2) one CTA per 64-key tile of one key/value head, looping over the query
// heads of its group and the query tiles that can see those keys; dK/dV stay
// in registers (summed over the group inside the CTA, no atomics), dQ is
// accumulated into the fp32 workspace, (3) dQ fp32 -> bf16 with the scale.
#include "common.cuh"
#include "kernels.h"

namespace uly {
namespace bwd_mma {

constexpr int BM = 64, BN = 64, kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdArgs {
  RankPtrs q, k, v, o, dO;
  RankPtrsFC lse;
  RankPtrsMut dq, dk, dv;
  const int32_t* cu;
  int num_seqs;
  int N, Hl, Hkvl, group;
  float scale, scale_log2;
  int rank_lo, nranks;
  int num_n_tiles;
  float* dq_acc;   // [P][N][Hl][D] fp32
  float* Dws;      // [P][Hl][N] fp32
};

template <int D>
ULY_DEV void load_tile(uint32_t s_base, const __nv_bfloat16* g, int row0, int N, int row_stride, int tid) {
  constexpr int CH = D / 8;
#pragma unroll
  for (int e = tid; e < 64 * CH; e += kThreads) {
    const int r = e / CH, c = e % CH;
    const int row = row0 + r;
    const bool ok = row < N;
    const __nv_bfloat16* src = g + static_cast<int64_t>(ok ? row : 0) * row_stride + c * 8;
    cp_async_16(s_base + swz<D>(r, c), src, ok);
  }
}

// (1) D_i = dO_i . O_i (fp32) and dq_acc = 0.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __grid_constant__ BwdArgs a) {
  constexpr int CH = D / 8;
  constexpr int RPB = 256 / CH;
  const int64_t rows_per_rank = static_cast<int64_t>(a.N) * a.Hl;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * RPB + threadIdx.x / CH;
  const int c = threadIdx.x % CH;
  float sum = 0.f;
  bool ok = e < rows_per_rank * a.nranks;
  int r = 0, i = 0, h = 0;
  if (ok) {
    const int rr = static_cast<int>(e / rows_per_rank);
    const int64_t rem = e - rr * rows_per_rank;
    i = static_cast<int>(rem / a.Hl);
    h = static_cast<int>(rem - static_cast<int64_t>(i) * a.Hl);
    r = a.rank_lo + rr;
    const int64_t off = (static_cast<int64_t>(i) * a.Hl + h) * D + c * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.o.p[r]) + off);
    const uint4 dv = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.dO.p[r]) + off);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 of = __bfloat1622float2(o2[k]);
      const float2 df = __bfloat1622float2(d2[k]);
      sum = fmaf(of.x, df.x, sum);
      sum = fmaf(of.y, df.y, sum);
    }
    float4* acc = reinterpret_cast<float4*>(a.dq_acc + static_cast<int64_t>(r) * rows_per_rank * D + off);
    acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int m = CH / 2; m >= 1; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
  if (ok && c == 0) a.Dws[static_cast<int64_t>(r) * rows_per_rank + static_cast<int64_t>(h) * a.N + i] = sum;
}

// (2) main backward kernel.
template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_mma_kernel(const __grid_constant__ BwdArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr uint32_t kTile = 64 * D * 2;
  const uint32_t sK = smem_u32(smem), sV = sK + kTile, sQ = sV + kTile, sdO = sQ + kTile, sdS = sdO + kTile;
  float* sLse = reinterpret_cast<float*>(smem + 4 * kTile + 64 * 64 * 2);
  float* sDv = sLse + 64;
  int* sStart = reinterpret_cast<int*>(sDv + 64);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.y * BN;                     // key tiles near the start carry the most rows
  const int g = blockIdx.x % a.Hkvl;
  const int r = a.rank_lo + blockIdx.x / a.Hkvl;
  const int N = a.N;
  const int qs = a.Hl * D, kvs = a.Hkvl * D;
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(a.k.p[r]) + g * D;
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(a.v.p[r]) + g * D;
  const int64_t rows_per_rank = static_cast<int64_t>(N) * a.Hl;
  float* dqa = a.dq_acc + static_cast<int64_t>(r) * rows_per_rank * D;
  const float* lse_r = a.lse.p[r];
  const float* D_r = a.Dws + static_cast<int64_t>(r) * rows_per_rank;

  load_tile<D>(sK, kb, n0, N, kvs, tid);
  load_tile<D>(sV, vb, n0, N, kvs, tid);
  cp_async_commit();

  const int kr_lo = n0 + warp * 16 + (lane >> 2), kr_hi = kr_lo + 8;
  const int m_end = doc_end_of(a.cu, a.num_seqs, min(n0 + BN - 1, N - 1), N);

  float dk_acc[D / 8][4], dv_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk_acc[i][e] = dv_acc[i][e] = 0.f;

  for (int hh = 0; hh < a.group; ++hh) {
    const int h = g * a.group + hh;
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q.p[r]) + h * D;
    const __nv_bfloat16* db = static_cast<const __nv_bfloat16*>(a.dO.p[r]) + h * D;
    for (int m0 = n0; m0 < m_end; m0 += BM) {
      __syncthreads();
      load_tile<D>(sQ, qb, m0, N, qs, tid);
      load_tile<D>(sdO, db, m0, N, qs, tid);
      cp_async_commit();
      if (tid < 64) {
        const int row = m0 + tid;
        if (row < N) {
          sLse[tid] = lse_r[static_cast<int64_t>(h) * N + row] * kLog2e;
          sDv[tid] = D_r[static_cast<int64_t>(h) * N + row];
          sStart[tid] = doc_start_of(a.cu, a.num_seqs, row);
        } else {
          sLse[tid] = INFINITY;   // exp2(s - inf) = 0: rows past N contribute nothing
          sDv[tid] = 0.f;
          sStart[tid] = 0;
        }
      }
      cp_async_wait<0>();
      __syncthreads();

      // S^T = K Q^T  (rows of S^T = this warp's 16 keys, columns = 64 query rows)
      float st[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) st[i][0] = st[i][1] = st[i][2] = st[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t ka[4];
        ldsm_x4(sK + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sQ + swz<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)), b0, b1, b2,
                  b3);
          mma_bf16_16816(st[2 * np], ka, b0, b1);
          mma_bf16_16816(st[2 * np + 1], ka, b2, b3);
        }
      }
      const int last_valid = min(BM - 1, N - 1 - m0);
      const bool need_mask = (m0 < n0 + BN) || (sStart[last_valid] > n0);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = e < 2 ? kr_lo : kr_hi;
          const int cl = nt * 8 + 2 * (lane & 3) + (e & 1);
          const int row = m0 + cl;
          const bool ok = !need_mask || (key <= row && key >= sStart[cl]);
          st[nt][e] = ok ? ex2_approx(st[nt][e] * a.scale_log2 - sLse[cl]) : 0.f;
        }
      }
      // dV += P^T dO
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(st[2 * kk][0], st[2 * kk][1]);
        pa[1] = pack_bf16x2(st[2 * kk][2], st[2 * kk][3]);
        pa[2] = pack_bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]);
        pa[3] = pack_bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3]);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sdO + swz<D>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), dp * 2 + (lane >> 4)), b0, b1,
                    b2, b3);
          mma_bf16_16816(dv_acc[2 * dp], pa, b0, b1);
          mma_bf16_16816(dv_acc[2 * dp + 1], pa, b2, b3);
        }
      }
      // dP^T = V dO^T
      float dpt[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) dpt[i][0] = dpt[i][1] = dpt[i][2] = dpt[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t va[4];
        ldsm_x4(sV + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), va[0], va[1], va[2], va[3]);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sdO + swz<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)), b0, b1, b2,
                  b3);
          mma_bf16_16816(dpt[2 * np], va, b0, b1);
          mma_bf16_16816(dpt[2 * np + 1], va, b2, b3);
        }
      }
      // dS^T = P^T (dP^T - D_i), kept in st
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int cl = nt * 8 + 2 * (lane & 3) + (e & 1);
          st[nt][e] = st[nt][e] * (dpt[nt][e] - sDv[cl]);
        }
      }
      // dK += dS^T Q ; stash dS^T (bf16, [key][row]) for the dQ product
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t da[4];
        da[0] = pack_bf16x2(st[2 * kk][0], st[2 * kk][1]);
        da[1] = pack_bf16x2(st[2 * kk][2], st[2 * kk][3]);
        da[2] = pack_bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]);
        da[3] = pack_bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3]);
        const int klo = warp * 16 + (lane >> 2);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sdS + swz<64>(klo, 2 * kk) + (lane & 3) * 4), "r"(da[0]));
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sdS + swz<64>(klo + 8, 2 * kk) + (lane & 3) * 4), "r"(da[1]));
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sdS + swz<64>(klo, 2 * kk + 1) + (lane & 3) * 4), "r"(da[2]));
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sdS + swz<64>(klo + 8, 2 * kk + 1) + (lane & 3) * 4),
                     "r"(da[3]));
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sQ + swz<D>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), dp * 2 + (lane >> 4)), b0, b1, b2,
                    b3);
          mma_bf16_16816(dk_acc[2 * dp], da, b0, b1);
          mma_bf16_16816(dk_acc[2 * dp + 1], da, b2, b3);
        }
      }
      __syncthreads();
      // dQ (this warp's 16 query rows) += dS K, 32 columns at a time, into the fp32 accumulator
      const int qr_lo = m0 + warp * 16 + (lane >> 2), qr_hi = qr_lo + 8;
#pragma unroll 1
      for (int dc = 0; dc < D / 32; ++dc) {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t aa[4];
          ldsm_x4_t(sdS + swz<64>(kk * 16 + (lane & 7) + ((lane >> 4) << 3), warp * 2 + ((lane >> 3) & 1)), aa[0],
                    aa[1], aa[2], aa[3]);
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sK + swz<D>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), dc * 4 + np * 2 + (lane >> 4)),
                      b0, b1, b2, b3);
            mma_bf16_16816(acc[2 * np], aa, b0, b1);
            mma_bf16_16816(acc[2 * np + 1], aa, b2, b3);
          }
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const int col = dc * 32 + nt * 8 + 2 * (lane & 3);
          if (qr_lo < N) {
            float* p = dqa + (static_cast<int64_t>(qr_lo) * a.Hl + h) * D + col;
            atomicAdd(p, acc[nt][0]);
            atomicAdd(p + 1, acc[nt][1]);
          }
          if (qr_hi < N) {
            float* p = dqa + (static_cast<int64_t>(qr_hi) * a.Hl + h) * D + col;
            atomicAdd(p, acc[nt][2]);
            atomicAdd(p + 1, acc[nt][3]);
          }
        }
      }
    }
  }

  __nv_bfloat16* dkb = static_cast<__nv_bfloat16*>(a.dk.p[r]) + g * D;
  __nv_bfloat16* dvb = static_cast<__nv_bfloat16*>(a.dv.p[r]) + g * D;
#pragma unroll
  for (int dt = 0; dt < D / 8; ++dt) {
    const int col = dt * 8 + 2 * (lane & 3);
    if (kr_lo < N) {
      const int64_t off = static_cast<int64_t>(kr_lo) * kvs + col;
      *reinterpret_cast<uint32_t*>(dkb + off) = pack_bf16x2(dk_acc[dt][0] * a.scale, dk_acc[dt][1] * a.scale);
      *reinterpret_cast<uint32_t*>(dvb + off) = pack_bf16x2(dv_acc[dt][0], dv_acc[dt][1]);
    }
    if (kr_hi < N) {
      const int64_t off = static_cast<int64_t>(kr_hi) * kvs + col;
      *reinterpret_cast<uint32_t*>(dkb + off) = pack_bf16x2(dk_acc[dt][2] * a.scale, dk_acc[dt][3] * a.scale);
      *reinterpret_cast<uint32_t*>(dvb + off) = pack_bf16x2(dv_acc[dt][2], dv_acc[dt][3]);
    }
  }
}

// (3) dQ = scale * dq_acc, fp32 -> bf16.
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const __grid_constant__ BwdArgs a, int D) {
  const int64_t per_rank = static_cast<int64_t>(a.N) * a.Hl * D / 8;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (e >= per_rank * a.nranks) return;
  const int rr = static_cast<int>(e / per_rank);
  const int64_t off = e - rr * per_rank;
  const int r = a.rank_lo + rr;
  const float4* src = reinterpret_cast<const float4*>(a.dq_acc + static_cast<int64_t>(r) * per_rank * 8) + off * 2;
  const float4 x = src[0], y = src[1];
  uint4 out;
  out.x = pack_bf16x2(x.x * a.scale, x.y * a.scale);
  out.y = pack_bf16x2(x.z * a.scale, x.w * a.scale);
  out.z = pack_bf16x2(y.x * a.scale, y.y * a.scale);
  out.w = pack_bf16x2(y.z * a.scale, y.w * a.scale);
  reinterpret_cast<uint4*>(a.dq.p[r])[off] = out;
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t stream) {
  {
    constexpr int RPB = 256 / (D / 8);
    const int64_t rows = static_cast<int64_t>(a.N) * a.Hl * a.nranks;
    bwd_pre_kernel<D><<<static_cast<unsigned>((rows + RPB - 1) / RPB), 256, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    const int smem = 4 * 64 * D * 2 + 64 * 64 * 2 + 3 * 64 * 4;
    cudaError_t e =
        cudaFuncSetAttribute(attn_bwd_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hkvl * a.nranks, a.num_n_tiles);
    attn_bwd_mma_kernel<D><<<grid, kThreads, smem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    const int64_t vecs = static_cast<int64_t>(a.N) * a.Hl * D / 8 * a.nranks;
    bwd_dq_convert_kernel<<<static_cast<unsigned>((vecs + 255) / 256), 256, 0, stream>>>(a, D);
    return cudaGetLastError();
  }
}

}  // namespace bwd_mma

size_t attn_bwd_workspace_bytes(int64_t N, int P, int Hl, int d) {
  using namespace bwd_mma;
  const size_t acc = static_cast<size_t>(P) * N * Hl * d * sizeof(float);
  const size_t dd = static_cast<size_t>(P) * N * Hl * sizeof(float);
  return acc + ((dd + 255) / 256) * 256;
}

cudaError_t launch_attn_bwd(const AttnShape& s, const void* const* q, const void* const* k, const void* const* v,
                            const void* const* o, const float* const* lse, const void* const* dO, void* const* dq,
                            void* const* dk, void* const* dv, void* workspace, cudaStream_t stream) {
  using namespace bwd_mma;
  BwdArgs a;
  memset(&a, 0, sizeof(a));
  for (int r = s.rank_lo; r < s.rank_hi; ++r) {
    a.q.p[r] = q[r];
    a.k.p[r] = k[r];
    a.v.p[r] = v[r];
    a.o.p[r] = o[r];
    a.dO.p[r] = dO[r];
    a.lse.p[r] = lse[r];
    a.dq.p[r] = dq[r];
    a.dk.p[r] = dk[r];
    a.dv.p[r] = dv[r];
  }
  a.cu = s.cu_seqlens;
  a.num_seqs = s.num_seqs;
  a.N = s.N;
  a.Hl = s.Hl;
  a.Hkvl = s.Hkvl;
  a.group = s.Hl / s.Hkvl;
  a.scale = s.scale;
  a.scale_log2 = s.scale * kLog2e;
  a.rank_lo = s.rank_lo;
  a.nranks = s.rank_hi - s.rank_lo;
  a.num_n_tiles = (s.N + BN - 1) / BN;
  // Workspace holds all P ranks (indexed by global rank) so rank ranges can be split freely.
  a.dq_acc = static_cast<float*>(workspace);
  a.Dws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                   static_cast<size_t>(s.P) * s.N * s.Hl * s.d * sizeof(float));
  return s.d == 64 ? launch_bwd_d<64>(a, stream) : launch_bwd_d<128>(a, stream);
}

}  // namespace uly
