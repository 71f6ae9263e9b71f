// Causal GQA (packed-varlen) flash-attention forward, warp-level mma.sync path.
//
// Computes, per rank r in range, per local query head h, per row i:
//   s_ij = scale * q_i.k_j  (j <= i, same document),  o_i = softmax(s_i) V,
//   lse_i = ln sum_j exp(s_ij)
// ("Compute attention locally" on each rank's heads over all positions --
// theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually Work?").
// One CTA = 64 query rows of one head (4 warps x 16 rows); K/V tiles of 64
// keys are double-buffered in shared memory with cp.async; the softmax is the
// online (running max / running sum) form in the log2 domain with fp32
// statistics; P is fed to the second GEMM straight from registers.
#include "common.cuh"
#include "kernels.h"

namespace uly {
namespace fwd_mma {

constexpr int BM = 64, BN = 64, kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct FwdArgs {
  RankPtrs q, k, v;
  RankPtrsMut o;
  RankPtrsF lse;
  const int32_t* cu;
  int num_seqs;
  int N, Hl, Hkvl, group;
  float scale_log2;
  int rank_lo;
  int num_m_tiles;
};

ULY_DEV float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
ULY_DEV void load_tile(uint32_t s_base, const __nv_bfloat16* g, int row0, int N, int row_stride, int tid) {
  constexpr int CH = D / 8;
#pragma unroll
  for (int e = tid; e < BM * CH; e += kThreads) {
    const int r = e / CH, c = e % CH;
    const int row = row0 + r;
    const bool ok = row < N;
    const __nv_bfloat16* src = g + static_cast<int64_t>(ok ? row : 0) * row_stride + c * 8;
    cp_async_16(s_base + swz<D>(r, c), src, ok);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_fwd_mma_kernel(const __grid_constant__ FwdArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = (a.num_m_tiles - 1 - static_cast<int>(blockIdx.y)) * BM;   // longest tiles first
  const int h = blockIdx.x % a.Hl;
  const int r = a.rank_lo + blockIdx.x / a.Hl;
  const int g = h / a.group;
  const int N = a.N;
  const int qs = a.Hl * D, kvs = a.Hkvl * D;
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q.p[r]) + h * D;
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(a.k.p[r]) + g * D;
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(a.v.p[r]) + g * D;

  constexpr uint32_t kTileBytes = BM * D * 2;
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + kTileBytes;          // 2 buffers
  const uint32_t sV = sK + 2 * kTileBytes;      // 2 buffers

  const int m_last = min(m0 + BM, N) - 1;
  const int kv_begin = doc_start_of(a.cu, a.num_seqs, m0);
  const int max_start = doc_start_of(a.cu, a.num_seqs, m_last);
  const int n_first = (kv_begin / BN) * BN;
  const int num_n = (m_last + 1 - n_first + BN - 1) / BN;

  const int r_lo = m0 + warp * 16 + (lane >> 2), r_hi = r_lo + 8;
  const int st_lo = doc_start_of(a.cu, a.num_seqs, min(r_lo, N - 1));
  const int st_hi = doc_start_of(a.cu, a.num_seqs, min(r_hi, N - 1));

  load_tile<D>(sQ, qb, m0, N, qs, tid);
  load_tile<D>(sK, kb, n_first, N, kvs, tid);
  load_tile<D>(sV, vb, n_first, N, kvs, tid);
  cp_async_commit();

  float o_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_i[2] = {-INFINITY, -INFINITY}, l_i[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];

  for (int it = 0; it < num_n; ++it) {
    const int buf = it & 1;
    if (it + 1 < num_n) {
      const int nn = n_first + (it + 1) * BN;
      load_tile<D>(sK + (buf ^ 1) * kTileBytes, kb, nn, N, kvs, tid);
      load_tile<D>(sV + (buf ^ 1) * kTileBytes, vb, nn, N, kvs, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(sQ + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2],
                qf[kk][3]);
    }
    const int n0 = n_first + it * BN;
    const uint32_t kbuf = sK + buf * kTileBytes, vbuf = sV + buf * kTileBytes;

    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbuf + swz<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)), b0, b1, b2,
                b3);
        mma_bf16_16816(s[2 * np], qf[kk], b0, b1);
        mma_bf16_16816(s[2 * np + 1], qf[kk], b2, b3);
      }
    }
    const bool need_mask = (n0 + BN - 1 > m0) || (n0 < max_start);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = n0 + nt * 8 + 2 * (lane & 3) + (e & 1);
        const int row = e < 2 ? r_lo : r_hi;
        const int st = e < 2 ? st_lo : st_hi;
        float x = s[nt][e] * a.scale_log2;
        if (need_mask && (col > row || col < st)) x = -INFINITY;
        s[nt][e] = x;
      }
    }
    float mx[2] = {m_i[0], m_i[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      mx[0] = fmaxf(mx[0], fmaxf(s[nt][0], s[nt][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[nt][2], s[nt][3]));
    }
    float base[2], alpha[2], rs[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
      base[i] = (mx[i] == -INFINITY) ? 0.f : mx[i];
      alpha[i] = ex2_approx(m_i[i] - base[i]);
      m_i[i] = mx[i];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = ex2_approx(s[nt][0] - base[0]);
      s[nt][1] = ex2_approx(s[nt][1] - base[0]);
      s[nt][2] = ex2_approx(s[nt][2] - base[1]);
      s[nt][3] = ex2_approx(s[nt][3] - base[1]);
      rs[0] += s[nt][0] + s[nt][1];
      rs[1] += s[nt][2] + s[nt][3];
    }
    l_i[0] = l_i[0] * alpha[0] + rs[0];
    l_i[1] = l_i[1] * alpha[1] + rs[1];
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      o_acc[dt][0] *= alpha[0];
      o_acc[dt][1] *= alpha[0];
      o_acc[dt][2] *= alpha[1];
      o_acc[dt][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbuf + swz<D>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), dp * 2 + (lane >> 4)), b0, b1,
                  b2, b3);
        mma_bf16_16816(o_acc[2 * dp], pa, b0, b1);
        mma_bf16_16816(o_acc[2 * dp + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_i[i] += __shfl_xor_sync(0xffffffffu, l_i[i], 1);
    l_i[i] += __shfl_xor_sync(0xffffffffu, l_i[i], 2);
  }
  const float inv0 = 1.f / l_i[0], inv1 = 1.f / l_i[1];
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.o.p[r]) + h * D;
#pragma unroll
  for (int dt = 0; dt < D / 8; ++dt) {
    const int col = dt * 8 + 2 * (lane & 3);
    if (r_lo < N)
      *reinterpret_cast<uint32_t*>(ob + static_cast<int64_t>(r_lo) * qs + col) =
          pack_bf16x2(o_acc[dt][0] * inv0, o_acc[dt][1] * inv0);
    if (r_hi < N)
      *reinterpret_cast<uint32_t*>(ob + static_cast<int64_t>(r_hi) * qs + col) =
          pack_bf16x2(o_acc[dt][2] * inv1, o_acc[dt][3] * inv1);
  }
  if ((lane & 3) == 0) {
    float* lb = a.lse.p[r] + static_cast<int64_t>(h) * N;
    if (r_lo < N) lb[r_lo] = (m_i[0] + lg2_approx(l_i[0])) * kLn2;
    if (r_hi < N) lb[r_hi] = (m_i[1] + lg2_approx(l_i[1])) * kLn2;
  }
}

template <int D>
cudaError_t launch_fwd_d(const AttnShape& s, const FwdArgs& a, cudaStream_t stream) {
  const int smem = 5 * BM * D * 2;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(s.Hl * (s.rank_hi - s.rank_lo), a.num_m_tiles);
  attn_fwd_mma_kernel<D><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fwd_mma

cudaError_t launch_attn_fwd(const AttnShape& s, const void* const* q, const void* const* k, const void* const* v,
                            void* const* o, float* const* lse, cudaStream_t stream) {
  using namespace fwd_mma;
  FwdArgs a;
  memset(&a, 0, sizeof(a));
  for (int r = s.rank_lo; r < s.rank_hi; ++r) {
    a.q.p[r] = q[r];
    a.k.p[r] = k[r];
    a.v.p[r] = v[r];
    a.o.p[r] = o[r];
    a.lse.p[r] = lse[r];
  }
  a.cu = s.cu_seqlens;
  a.num_seqs = s.num_seqs;
  a.N = s.N;
  a.Hl = s.Hl;
  a.Hkvl = s.Hkvl;
  a.group = s.Hl / s.Hkvl;
  a.scale_log2 = s.scale * kLog2e;
  a.rank_lo = s.rank_lo;
  a.num_m_tiles = (s.N + BM - 1) / BM;
  return s.d == 64 ? launch_fwd_d<64>(s, a, stream) : launch_fwd_d<128>(s, a, stream);
}

}  // namespace uly
