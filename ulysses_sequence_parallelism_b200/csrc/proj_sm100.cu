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
// Their gradients are the same kernel with other operand views (backward of
// the block; the pages train through it):
//   dO  = dY W_o         (A: dY sequence shards; B: W_o read N-major; out:
//                         head shards -- the seq -> head permute of dO is gone)
//   dW_o = dY^T O        (A: dY read M-major, reduction over all tokens; B: O
//                         read N-major from the head shards)
//   dX  = [dQ|dK|dV] W_qkv (A gathered from the three head shards; B: W_qkv
//                         read N-major; out: sequence shards -- the head -> seq
//                         permute of dQ, dK, dV is gone)
//   dW_qkv = [dQ|dK|dV]^T X (A: head shards read M-major; B: X read N-major)
// One CTA computes a 128 x 256 output tile over the whole reduction:
//   warp 0 : TMA producer (A 128 x 64 and B 256 x 64 per stage, 4 stages);
//            K-major tiles are one box, M/N-major tiles are 64-wide boxes
//   warp 1 : MMA issuer, tcgen05.mma M=128 N=256 K=16 (SS), fp32 accumulator
//            in TMEM columns [0, 256)
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

// Operand views: where a 64-deep slab of an A (128 rows) or B (256 rows) tile comes from.
enum Src : int {
  SEQ_K = 0,    // rows = tokens of one sequence shard, reduction = features (contiguous)
  HEAD_K = 1,   // rows = tokens, reduction = features gathered from head shards
  PLAIN_K = 2,  // rows = matrix rows, reduction = matrix columns (contiguous)
  PLAIN_MN = 3, // rows = matrix columns (contiguous), reduction = matrix rows
  SEQ_MN = 4,   // rows = features of sequence shards (contiguous), reduction = tokens
  HEAD_MN = 5,  // rows = features of head shards (contiguous), reduction = tokens
};
enum Out : int { OUT_HEADS = 0, OUT_SEQ = 1, OUT_PLAIN = 2, OUT_PLAIN_F32_ADD = 3 };

struct Layout {
  static constexpr uint32_t kA = BM * BK * 2;          // 16 KB
  static constexpr uint32_t kB = BN * BK * 2;          // 32 KB
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kBars = NS * kStage;       // full[NS], empty[NS], acc_full
  static constexpr int kNumBars = 2 * NS + 1;
  static constexpr uint32_t kSlot = kBars + kNumBars * 8;
  static constexpr uint32_t kAlloc = kSlot + 16 + 1024;
};

struct GemmArgs {
  CUtensorMap ta[3][kMaxRanks];   // A maps: [tensor][rank] (head shards) or [0][shard] / [0][0]
  CUtensorMap tb[3][kMaxRanks];   // B maps, same convention
  RankPtrsMut out[3];             // OUT_HEADS: [tensor].p[rank]; OUT_SEQ: [0].p[shard]; OUT_PLAIN: [0].p[0]
  int a_src, b_src, out_kind, a_mn, b_mn;
  int tok_m;                      // 1: output rows are tokens (tile = shard, row); 0: rows are features
  int k_chunk;                    // > 0: blockIdx.z takes reduction range [z*k_chunk, +k_chunk) (split-K)
  int n_loc, P, K, n_out, H, H_kv, d;
  int m_tiles;                    // tok_m: row tiles per shard
};

// Feature f of the concatenated heads (H query heads, then H_kv key, then H_kv
// value heads, d each) -> tensor, owning rank, column within that head shard.
ULY_DEV void feature_loc(const GemmArgs& a, int f, int& tensor, int& rank, int& col, int& hl) {
  int head = f / a.d;
  const int c = f - head * a.d;
  tensor = 0;
  hl = a.H / a.P;
  if (head >= a.H + a.H_kv) { tensor = 2; head -= a.H + a.H_kv; hl = a.H_kv / a.P; }
  else if (head >= a.H) { tensor = 1; head -= a.H; hl = a.H_kv / a.P; }
  rank = head / hl;
  col = (head - rank * hl) * a.d + c;
}

// Issue the loads of one 64-deep slab of a tile of ROWS rows starting at r0
// (tokens: shard p / row s0 / global t0) into dst.
template <int SRC, int ROWS>
ULY_DEV void load_slab(const GemmArgs& a, const CUtensorMap (*maps)[kMaxRanks], uint32_t dst, int r0, int p, int s0,
                       int k0, uint32_t bar) {
  if constexpr (SRC == SEQ_K) {
    tma_load_2d_w(dst, &maps[0][p], bar, k0, s0);
  } else if constexpr (SRC == HEAD_K) {
    int t, q, x, hl;
    feature_loc(a, k0, t, q, x, hl);
    tma_load_2d_w(dst, &maps[t][q], bar, x, p * a.n_loc + s0);
  } else if constexpr (SRC == PLAIN_K) {
    tma_load_2d_w(dst, &maps[0][0], bar, k0, r0);
  } else if constexpr (SRC == PLAIN_MN) {
#pragma unroll
    for (int i = 0; i < ROWS / 64; ++i) tma_load_2d_w(dst + 8192u * i, &maps[0][0], bar, r0 + 64 * i, k0);
  } else if constexpr (SRC == SEQ_MN) {
    const int sh = k0 / a.n_loc;
#pragma unroll
    for (int i = 0; i < ROWS / 64; ++i)
      tma_load_2d_w(dst + 8192u * i, &maps[0][sh], bar, r0 + 64 * i, k0 - sh * a.n_loc);
  } else {   // HEAD_MN
#pragma unroll
    for (int i = 0; i < ROWS / 64; ++i) {
      int t, q, x, hl;
      feature_loc(a, r0 + 64 * i, t, q, x, hl);
      tma_load_2d_w(dst + 8192u * i, &maps[t][q], bar, x, k0);
    }
  }
}

__host__ __device__ constexpr bool mn_major(int src) { return src == PLAIN_MN || src == SEQ_MN || src == HEAD_MN; }

// One instantiation per (A view, B view, output) in use: every view and
// descriptor constant is known at compile time.
template <int ASRC, int BSRC, int OUTK>
__global__ void __launch_bounds__(kThreads, 1) proj_kernel(const __grid_constant__ GemmArgs a) {
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
  int p = 0, s0 = 0, m0 = 0;
  if (a.tok_m) {
    p = blockIdx.y / a.m_tiles;                          // sequence shard of this tile's tokens
    s0 = (blockIdx.y - p * a.m_tiles) * BM;              // first row within the shard
  } else {
    m0 = blockIdx.y * BM;                                // first output feature row
  }
  // Reduction steps of this CTA: all of K, or one split-K chunk of it. With
  // the split index slowest in the grid, the CTAs resident together share
  // one chunk of the token-long operands, which then stays in L2.
  int kt0 = 0, KT = a.K / BK;
  if (a.k_chunk > 0) {
    kt0 = blockIdx.z * (a.k_chunk / BK);
    KT = min(a.K / BK - kt0, a.k_chunk / BK);
  }

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
    int kt = 0;
    for (; kt < KT; ++kt) {
      const int s = kt % NS;
      if (!mbar_wait_warp(empty(s), ((kt / NS) & 1) ^ 1, kErrProj, 0x100 + s)) break;
      const uint32_t st = sbase + s * L::kStage;
      mbar_arrive_expect_tx_w(full(s), L::kStage);
      load_slab<ASRC, BM>(a, a.ta, st, m0, p, s0, (kt0 + kt) * BK, full(s));
      load_slab<BSRC, BN>(a, a.tb, st + L::kA, n0, p, s0, (kt0 + kt) * BK, full(s));
    }
    for (int k = kt > NS ? kt - NS : 0; k < kt; ++k)
      mbar_wait_drain_w(full(k % NS), (k / NS) & 1, kErrProj, 0x1F0);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // K-major tile: one 128-byte-swizzled box, K step = 32 bytes along the row.
    // M/N-major tile: 64-element atoms 8 KB apart (LBO), K step = 16 rows = 2 KB.
    constexpr bool AMN = mn_major(ASRC), BMN = mn_major(BSRC);
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, AMN ? 1 : 0, BMN ? 1 : 0);
    const uint64_t dA0 = smem_desc_sw128(sbase, AMN ? 8192 : 16, 1024);
    const uint64_t dB0 = smem_desc_sw128(sbase + L::kA, BMN ? 8192 : 16, 1024);
    constexpr uint32_t ka = AMN ? 2048 : 32, kb = BMN ? 2048 : 32;
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % NS;
      if (!mbar_wait_warp(full(s), (kt / NS) & 1, kErrProj, 0x200 + s)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        mma_ss_w(tmem, desc_adv(dA0, s * L::kStage + kk * ka), desc_adv(dB0, s * L::kStage + kk * kb), idesc,
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
      const int64_t t = static_cast<int64_t>(p) * a.n_loc + s0 + row;   // global token (tok_m)
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + loff + c * 32, v);
        tmem_wait_ld();
        const int f = n0 + c * 32;                       // first output column of this chunk (inside one head)
        if constexpr (OUTK == OUT_PLAIN_F32_ADD) {
          // fp32 partial sum of this split-K chunk, added in L2
          float* dstf = static_cast<float*>(a.out[0].p[0]) + static_cast<int64_t>(m0 + row) * a.n_out + f;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dstf + 4 * e),
                         "f"(__uint_as_float(v[4 * e])), "f"(__uint_as_float(v[4 * e + 1])),
                         "f"(__uint_as_float(v[4 * e + 2])), "f"(__uint_as_float(v[4 * e + 3]))
                         : "memory");
          continue;
        }
        uint4 o4[4];
        uint32_t* ow = reinterpret_cast<uint32_t*>(o4);
#pragma unroll
        for (int e = 0; e < 16; ++e) ow[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        __nv_bfloat16* dst;
        if constexpr (OUTK == OUT_HEADS) {
          int tn, q, col, hl;
          feature_loc(a, f, tn, q, col, hl);
          dst = static_cast<__nv_bfloat16*>(a.out[tn].p[q]) + t * hl * a.d + col;
        } else if constexpr (OUTK == OUT_SEQ) {
          dst = static_cast<__nv_bfloat16*>(a.out[0].p[p]) + static_cast<int64_t>(s0 + row) * a.n_out + f;
        } else {
          dst = static_cast<__nv_bfloat16*>(a.out[0].p[0]) + static_cast<int64_t>(m0 + row) * a.n_out + f;
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

// Maps of one operand. kind K-major: box rows = tile rows; M/N-major: 64.
// bufs[t][r]: head shards (r < P) of tensor t, or sequence shards, or bufs[0][0].
bool encode_operand(bwd_sm100::EncodeTiledFn enc, CUtensorMap (*maps)[kMaxRanks], int src, int tile_rows,
                    const void* const* const bufs[3], int ntensors, int64_t N, int P, int64_t row_elems_plain,
                    int64_t rows_plain, const int hx[3], int d, int64_t seq_cols) {
  const int box = (src == SEQ_K || src == HEAD_K || src == PLAIN_K) ? tile_rows : 64;
  if (src == PLAIN_K || src == PLAIN_MN) return bwd_sm100::encode(enc, &maps[0][0], bufs[0][0], rows_plain,
                                                                  row_elems_plain, box);
  if (src == SEQ_K || src == SEQ_MN) {
    for (int r = 0; r < P; ++r)
      if (!bwd_sm100::encode(enc, &maps[0][r], bufs[0][r], N / P, seq_cols, box)) return false;
    return true;
  }
  for (int t = 0; t < ntensors; ++t)
    for (int r = 0; r < P; ++r)
      if (!bwd_sm100::encode(enc, &maps[t][r], bufs[t][r], N, static_cast<int64_t>(hx[t] / P) * d, box))
        return false;
  return true;
}

}  // namespace proj_sm100

cudaError_t launch_proj_gemm(const ProjGemm& g, cudaStream_t stream) {
  using namespace proj_sm100;
  bwd_sm100::EncodeTiledFn enc = bwd_sm100::get_encode();
  if (enc == nullptr) return cudaErrorNotSupported;
  GemmArgs* a = new GemmArgs;       // ~13 KB of tensor maps: keep it off the caller's stack
  memset(a, 0, sizeof(*a));
  a->a_src = g.a_src;
  a->b_src = g.b_src;
  a->out_kind = g.out_kind;
  a->a_mn = (g.a_src == PLAIN_MN || g.a_src == SEQ_MN || g.a_src == HEAD_MN) ? 1 : 0;
  a->b_mn = (g.b_src == PLAIN_MN || g.b_src == SEQ_MN || g.b_src == HEAD_MN) ? 1 : 0;
  a->tok_m = g.tok_m;
  a->k_chunk = g.k_chunk;
  a->n_loc = static_cast<int>(g.N / g.P);
  a->P = g.P;
  a->K = g.K;
  a->n_out = g.n_out;
  a->H = g.H;
  a->H_kv = g.H_kv;
  a->d = g.d;
  a->m_tiles = a->n_loc / BM;
  const int hx[3] = {g.H, g.H_kv, g.H_kv};
  bool ok = encode_operand(enc, a->ta, g.a_src, BM, g.a_bufs, g.a_ntensors, g.N, g.P, g.a_plain_cols,
                           g.a_plain_rows, hx, g.d, g.a_seq_cols) &&
            encode_operand(enc, a->tb, g.b_src, BN, g.b_bufs, g.b_ntensors, g.N, g.P, g.b_plain_cols,
                           g.b_plain_rows, hx, g.d, g.b_seq_cols);
  if (!ok) {
    delete a;
    return cudaErrorInvalidValue;
  }
  for (int t = 0; t < 3; ++t)
    for (int r = 0; r < kMaxRanks; ++r) a->out[t].p[r] = g.out[t][r];
  // the (A view, B view, output) combinations the entry points use
  void (*kern)(GemmArgs) = nullptr;
  if (g.a_src == SEQ_K && g.b_src == PLAIN_K && g.out_kind == OUT_HEADS) kern = proj_kernel<SEQ_K, PLAIN_K, OUT_HEADS>;
  else if (g.a_src == HEAD_K && g.b_src == PLAIN_K && g.out_kind == OUT_SEQ) kern = proj_kernel<HEAD_K, PLAIN_K, OUT_SEQ>;
  else if (g.a_src == SEQ_K && g.b_src == PLAIN_MN && g.out_kind == OUT_HEADS) kern = proj_kernel<SEQ_K, PLAIN_MN, OUT_HEADS>;
  else if (g.a_src == SEQ_MN && g.b_src == HEAD_MN && g.out_kind == OUT_PLAIN_F32_ADD)
    kern = proj_kernel<SEQ_MN, HEAD_MN, OUT_PLAIN_F32_ADD>;
  else if (g.a_src == HEAD_K && g.b_src == PLAIN_MN && g.out_kind == OUT_SEQ) kern = proj_kernel<HEAD_K, PLAIN_MN, OUT_SEQ>;
  else if (g.a_src == HEAD_MN && g.b_src == SEQ_MN && g.out_kind == OUT_PLAIN_F32_ADD)
    kern = proj_kernel<HEAD_MN, SEQ_MN, OUT_PLAIN_F32_ADD>;
  cudaError_t e = kern == nullptr ? cudaErrorInvalidValue : cudaSuccess;
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::kAlloc);
  if (e == cudaSuccess) {
    const int splits = g.k_chunk > 0 ? (g.K + g.k_chunk - 1) / g.k_chunk : 1;
    dim3 grid(g.n_out / BN, g.tok_m ? g.P * a->m_tiles : g.m_rows / BM, splits);
    kern<<<grid, kThreads, Layout::kAlloc, stream>>>(*a);
    e = cudaGetLastError();
  }
  delete a;
  return e;
}

}  // namespace uly
