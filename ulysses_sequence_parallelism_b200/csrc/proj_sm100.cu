// QKV and output projections with the Ulysses all-to-alls folded into the GEMMs
// (sm_100a: TMA-fed 128-byte-swizzled tiles, tcgen05 MMA into TMEM).
//
// The pages put a projection on each side of the exchange: every rank projects
// Q, K, V for its own chunk of tokens before the first all-to-all, and projects
// the attention output on its shard after the second (theaicatchup.com, "How
// Does Ulysses Sequence Parallelism Actually Work?"; contenidos2-1ml.pages.dev,
// "¿Qué es Ulysses y por qué importa?"). Here those GEMMs absorb the exchange:
//   QKV : [Q | K | V] = X W_qkv^T per token (X: sequence shards [N/P, hidden];
//         W_qkv: [(H + 2 H_kv) d, hidden]); the epilogue stores each output
//         column straight into the head shard of the rank that owns its head,
//         so the seq -> head permute never runs.
//   OUT : Y = O W_o^T per token (W_o: [hidden, H d]); the A operand (O in
//         sequence order) is fetched tile by tile straight from the head shards
//         ([N, H/P, d] per rank: a 64-column slice of one head of one rank), so
//         the head -> seq permute never runs; Y lands in the sequence shards.
// One CTA computes a 128-token x 256-column tile over the whole reduction:
//   warp 0 : TMA producer (A 128 x 64 and B 256 x 64 per stage, 4 stages)
//   warp 1 : MMA issuer, tcgen05.mma M=128 N=256 K=16 (SS, both K-major),
//            fp32 accumulator in TMEM columns [0, 256)
//   warps 2-5: epilogue, one thread per row (TMEM lane), bf16 (round to
//            nearest even) stores.
// Every mbarrier wait is bounded and reports into the library error word.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace uly {
namespace proj_sm100 {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int NS = 4;
constexpr int kThreads = 192;
constexpr uint32_t kErrProj = 4u;

struct Layout {
  static constexpr uint32_t kA = BM * BK * 2;          // 16 KB
  static constexpr uint32_t kB = BN * BK * 2;          // 32 KB
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kBars = NS * kStage;       // full[NS], empty[NS], acc_full
  static constexpr int kNumBars = 2 * NS + 1;
  static constexpr uint32_t kSlot = kBars + kNumBars * 8;
  static constexpr uint32_t kAlloc = kSlot + 16 + 1024;
};

struct ProjArgs {
  CUtensorMap ta[kMaxRanks];   // QKV: X shard p [N/P, hidden]; OUT: O head shard q [N, Hl*d]
  CUtensorMap tb;              // W [n_out, K]
  RankPtrsMut out0, out1, out2;   // QKV: Q, K, V head shards per rank; OUT: Y sequence shards
  int mode;                    // 0 = QKV, 1 = OUT
  int n_loc, P, K, n_out;
  int H, H_kv, d;
  int m_tiles;                 // n_loc / BM
};

__global__ void __launch_bounds__(kThreads, 1) proj_kernel(const __grid_constant__ ProjArgs a) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t bars = sbase + L::kBars;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (NS + s); };
  const uint32_t acc_full = bars + 8u * (2 * NS);
  volatile uint32_t* slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int p = blockIdx.y / a.m_tiles;                  // sequence shard of this tile's tokens
  const int s0 = (blockIdx.y - p * a.m_tiles) * BM;      // first row within the shard
  const int KT = a.K / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bars + 8u * i, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kSlot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const int Hl = a.H / a.P;
    int kt = 0;
    for (; kt < KT; ++kt) {
      const int s = kt % NS;
      if (!mbar_wait_warp(empty(s), ((kt / NS) & 1) ^ 1, kErrProj, 0x100 + s)) break;
      const uint32_t st = sbase + s * L::kStage;
      mbar_arrive_expect_tx_w(full(s), L::kStage);
      if (a.mode == 0) {
        tma_load_2d_w(st, &a.ta[p], full(s), kt * BK, s0);
      } else {
        // features [64 kt, 64 kt + 64) of O are columns of one head of one rank
        const int f = kt * BK;
        const int h = f / a.d, c0 = f - h * a.d;
        const int q = h / Hl, j = h - q * Hl;
        tma_load_2d_w(st, &a.ta[q], full(s), j * a.d + c0, p * a.n_loc + s0);
      }
      tma_load_2d_w(st + L::kA, &a.tb, full(s), kt * BK, n0);
    }
    for (int k = kt > NS ? kt - NS : 0; k < kt; ++k)
      mbar_wait_drain_w(full(k % NS), (k / NS) & 1, kErrProj, 0x1F0);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
    const uint64_t dA0 = smem_desc_sw128(sbase, 16, 1024);
    const uint64_t dB0 = smem_desc_sw128(sbase + L::kA, 16, 1024);
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % NS;
      if (!mbar_wait_warp(full(s), (kt / NS) & 1, kErrProj, 0x200 + s)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        mma_ss_w(tmem, desc_adv(dA0, s * L::kStage + kk * 32), desc_adv(dB0, s * L::kStage + kk * 32), idesc,
                 (kt > 0 || kk > 0) ? 1u : 0u);
      mma_commit_w(empty(s));
    }
    mma_commit_w(acc_full);
    mbar_wait_drain_w(acc_full, 0, kErrProj, 0x250);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int lq = warp & 3;                             // TMEM lane quadrant of this warp
    const int row = 32 * lq + lane;
    const uint32_t loff = static_cast<uint32_t>(32 * lq) << 16;
    if (mbar_wait_warp(acc_full, 0, kErrProj, 0x300)) {
      tc_fence_after();
      const int64_t t = static_cast<int64_t>(p) * a.n_loc + s0 + row;   // global token
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + loff + c * 32, v);
        tmem_wait_ld();
        uint4 o4[4];
        uint32_t* ow = reinterpret_cast<uint32_t*>(o4);
#pragma unroll
        for (int e = 0; e < 16; ++e) ow[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        const int f = n0 + c * 32;                       // first output column of this chunk
        __nv_bfloat16* dst;
        if (a.mode == 0) {
          int tensor = 0, head = f / a.d;
          const int dim = f - head * a.d;
          int hx = a.H;
          if (head >= a.H + a.H_kv) { tensor = 2; head -= a.H + a.H_kv; hx = a.H_kv; }
          else if (head >= a.H) { tensor = 1; head -= a.H; hx = a.H_kv; }
          const int hl = hx / a.P, q = head / hl, j = head - q * hl;
          void* base = tensor == 0 ? a.out0.p[q] : (tensor == 1 ? a.out1.p[q] : a.out2.p[q]);
          dst = static_cast<__nv_bfloat16*>(base) + (t * hl + j) * a.d + dim;
        } else {
          dst = static_cast<__nv_bfloat16*>(a.out0.p[p]) + static_cast<int64_t>(s0 + row) * a.n_out + f;
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int e = 0; e < 4; ++e) d4[e] = o4[e];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

}  // namespace proj_sm100

cudaError_t launch_proj(int mode, const void* const* a_bufs, const void* w, void* const* out0, void* const* out1,
                        void* const* out2, int64_t N, int P, int H, int H_kv, int d, int hidden,
                        cudaStream_t stream) {
  using namespace proj_sm100;
  bwd_sm100::EncodeTiledFn enc = bwd_sm100::get_encode();
  if (enc == nullptr) return cudaErrorNotSupported;
  ProjArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = mode;
  a.n_loc = static_cast<int>(N / P);
  a.P = P;
  a.H = H;
  a.H_kv = H_kv;
  a.d = d;
  a.m_tiles = a.n_loc / BM;
  if (mode == 0) {
    a.K = hidden;
    a.n_out = (H + 2 * H_kv) * d;
    for (int r = 0; r < P; ++r) {
      if (!bwd_sm100::encode(enc, &a.ta[r], a_bufs[r], a.n_loc, hidden, BM)) return cudaErrorInvalidValue;
      a.out0.p[r] = out0[r];
      a.out1.p[r] = out1[r];
      a.out2.p[r] = out2[r];
    }
  } else {
    a.K = H * d;
    a.n_out = hidden;
    for (int r = 0; r < P; ++r) {
      if (!bwd_sm100::encode(enc, &a.ta[r], a_bufs[r], N, static_cast<int64_t>(H / P) * d, BM))
        return cudaErrorInvalidValue;
      a.out0.p[r] = out0[r];
    }
  }
  if (!bwd_sm100::encode(enc, &a.tb, w, a.n_out, a.K, BN)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_out / BN, P * a.m_tiles);
  proj_kernel<<<grid, kThreads, Layout::kAlloc, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace uly
