// Causal GQA (packed-varlen) flash-attention backward for sm_100a: tcgen05 MMA
// with TMEM accumulators, TMA-fed shared-memory tiles, warp-specialised.
//
// Gradient of the forward (the pages train through the layer but do not write
// its backward; this is softmax-attention calculus), with scale = softmax scale:
//   P_ij = exp(s_ij - lse_i),  D_i = dO_i . O_i
//   dV_j = sum_i P_ij dO_i,    dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - D_i)
//   dK_j = scale sum_i dS_ij q_i,   dQ_i = scale sum_j dS_ij k_j
// dK/dV of a key/value head are summed over the H/H_kv query heads reading it.
//
// With deterministic == 1 (or head dim 64): three launches, no atomics anywhere:
//  1. prep : D_i and lse_i*log2(e) per (rank, head, row) into a workspace
//            padded to a multiple of 128 rows (padding: lse = +inf, D = 0, so
//            padded rows contribute exactly zero).
//  2. dkdv : one CTA per 128-key block of one key/value head. K and V stay in
//            shared memory; the CTA streams 64-row blocks of Q and dO (every
//            query head of the group, every row that can see these keys):
//              S^T = K Q^T, dP^T = V dO^T          (SS MMAs, double-buffered)
//              P^T, dS^T elementwise (one thread per key row), bf16 into TMEM
//              dV += P^T dO,  dK += dS^T Q         (TS MMAs into TMEM)
//  3. dq   : one CTA per 128-row block of one query head. Q and dO stay in
//            shared memory; the CTA streams 128-key blocks of K and V:
//              S = Q K^T, dP = dO V^T; dS elementwise (one thread per row,
//              the two warpgroups on the two key halves); dQ += dS K (TS MMA).
// S and dP are recomputed in (3): 7 block GEMMs instead of 5, in exchange for
// no fp32 atomics, no dQ accumulator traffic and a bit-reproducible result.
// With deterministic == 0 and head dim 128, the one-pass kernel
// (attn_bwd_onepass_sm100.cuh) replaces (2) and (3): 5 block GEMMs, dQ summed
// in fp32 by L2 vector reductions into a workspace accumulator.
// Layouts: as in the forward, seq == 0 reads and writes rank r's head shards
// ([N, Hx/P, d]); seq == 1 (the fused path) maps the sequence shards
// ([N/P, Hx, d], N/P a multiple of 128) and addresses rank r's heads as the
// column slice at r*Hx/P*d, so no permute runs before or after.
// Warp roles in 2 and 3: warps 0-3 / 4-7 elementwise, warp 8 TMA producer,
// warp 9 MMA issuer (TMA and MMA warps run converged; one elected lane issues).
// Every mbarrier wait is bounded and reports into the library error word.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace uly {
namespace bwd_sm100 {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr int NST = 4;          // ring stages
constexpr int SB = 64;          // streamed block (rows in dkdv, keys in dq)
constexpr int TB = 128;         // stationary block (keys in dkdv, rows in dq)
constexpr float kLog2e = 1.4426950408889634f;

ULY_DEV float u2f(uint32_t x) { return __uint_as_float(x); }
ULY_DEV float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}


// ====================================================================== prep
struct PrepArgs {
  RankPtrs o, dO;
  RankPtrsFC lse;
  float* lse2;    // [P][Hl][Npad]
  float* Dv;      // [P][Hl][Npad]
  int N, Npad, Hl, rank_lo, nranks;
  int seq, n_loc, P;
};

template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __grid_constant__ PrepArgs a) {
  constexpr int CH = D / 8;            // 16-byte chunks per head row
  constexpr int RPB = 256 / CH;
  const int64_t rows_per_rank = static_cast<int64_t>(a.Npad) * a.Hl;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * RPB + threadIdx.x / CH;
  const int c = threadIdx.x % CH;
  const bool ok = e < rows_per_rank * a.nranks;
  int r = 0, i = 0, h = 0;
  float sum = 0.f;
  if (ok) {
    const int rr = static_cast<int>(e / rows_per_rank);
    const int64_t rem = e - rr * rows_per_rank;
    i = static_cast<int>(rem / a.Hl);
    h = static_cast<int>(rem - static_cast<int64_t>(i) * a.Hl);
    r = a.rank_lo + rr;
    if (i < a.N) {
      int buf = r;
      int64_t off = (static_cast<int64_t>(i) * a.Hl + h) * D + c * 8;
      if (a.seq) {
        buf = i / a.n_loc;
        off = (static_cast<int64_t>(i - buf * a.n_loc) * (a.Hl * a.P) + r * a.Hl + h) * D + c * 8;
      }
      const uint4 ov = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.o.p[buf]) + off);
      const uint4 dv = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.dO.p[buf]) + off);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 of = __bfloat1622float2(o2[k]);
        const float2 df = __bfloat1622float2(d2[k]);
        sum = fmaf(of.x, df.x, sum);
        sum = fmaf(of.y, df.y, sum);
      }
    }
  }
#pragma unroll
  for (int m = CH / 2; m >= 1; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
  if (ok && c == 0) {
    const int64_t idx = (static_cast<int64_t>(r) * a.Hl + h) * a.Npad + i;
    if (i < a.N) {
      a.Dv[idx] = sum;
      a.lse2[idx] = a.lse.p[r][static_cast<int64_t>(h) * a.N + i] * kLog2e;
    } else {
      a.Dv[idx] = 0.f;
      a.lse2[idx] = INFINITY;
    }
  }
}

// ====================================================================== dK, dV
struct DkdvArgs {
  CUtensorMap tq[kMaxRanks];    // box 64 cols x SB rows (TB rows for the one-pass kernel)
  CUtensorMap tdo[kMaxRanks];   // box 64 cols x SB rows (TB rows for the one-pass kernel)
  CUtensorMap tk[kMaxRanks];    // box 64 cols x TB rows
  CUtensorMap tv[kMaxRanks];    // box 64 cols x TB rows
  RankPtrsMut dk, dv;
  const float* lse2;
  const float* Dv;
  float* dqacc;                 // one-pass kernel only: fp32 dQ accumulator
  const int32_t* cu;
  int num_seqs;
  int N, Npad, Hl, Hkvl, group;
  float scale, scale_log2;
  int rank_lo;
  int seq, n_loc, P;
  int kb_fast;                  // one-pass kernel only: blockIdx.x is the key block (else the kv head)
  int qdo_seq;                  // one-pass kernel only: tq/tdo map sequence shards (else head shards)
};

template <int D>
struct DkdvLayout {
  static constexpr uint32_t kKV = TB * D * 2;         // one stationary K or V tile
  static constexpr uint32_t kBlk = SB * D * 2;        // one streamed Q or dO block
  static constexpr uint32_t kK = 0, kV = kKV;
  static constexpr uint32_t kRing = 2 * kKV;          // stage s: Q at +0, dO at +kBlk
  static constexpr uint32_t kVec = kRing + NST * 2 * kBlk;   // stage s: lse2 at +0, D at +256
  static constexpr uint32_t kBars = kVec + NST * 512;
  // kv_full, st_full[NST], st_empty[NST], s_full[2], dp_full[2], p_full[2], ds_full[2], dv_done[2],
  // dk_done[2], acc_done
  static constexpr int kNumBars = 1 + 2 * NST + 12 + 1;
  static constexpr uint32_t kSlot = kBars + kNumBars * 8;
  static constexpr uint32_t kAlloc = kSlot + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dkdv_kernel(const __grid_constant__ DkdvArgs a) {
  using L = DkdvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t bars = sbase + L::kBars;
  const uint32_t kv_full = bars;
  auto st_full = [&](int s) { return bars + 8u * (1 + s); };
  auto st_empty = [&](int s) { return bars + 8u * (1 + NST + s); };
  auto s_full = [&](int b) { return bars + 8u * (1 + 2 * NST + b); };
  auto dp_full = [&](int b) { return bars + 8u * (3 + 2 * NST + b); };
  auto p_full = [&](int b) { return bars + 8u * (5 + 2 * NST + b); };
  auto ds_full = [&](int b) { return bars + 8u * (7 + 2 * NST + b); };
  auto dv_done = [&](int b) { return bars + 8u * (9 + 2 * NST + b); };
  auto dk_done = [&](int b) { return bars + 8u * (11 + 2 * NST + b); };
  const uint32_t acc_done = bars + 8u * (13 + 2 * NST);
  volatile uint32_t* slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % a.Hkvl;
  const int r = a.rank_lo + blockIdx.x / a.Hkvl;
  const int N = a.N;
  const int n0 = blockIdx.y * TB;                      // key blocks near the start carry the most rows
  const int n_last = min(n0 + TB, N) - 1;
  const int doc_end_first = doc_end_of(a.cu, a.num_seqs, n0, N);
  const int m_end = doc_end_of(a.cu, a.num_seqs, n_last, N);
  const int rb_lo = n0 / SB;
  const int nrb = (m_end + SB - 1) / SB - rb_lo;
  const int T = a.group * nrb;                          // streamed iterations

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bars + 8u * i, 1);
    mbar_init(p_full(0), 128);
    mbar_init(p_full(1), 128);
    mbar_init(ds_full(0), 128);
    mbar_init(ds_full(1), 128);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sbase + L::kSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t tDV = tmem, tDK = tmem + D;
  auto tS = [&](int b) { return tmem + 256u + 128u * b; };
  auto tDP = [&](int b) { return tmem + 256u + 128u * b + 64u; };

  if (warp == kTmaWarp) {
    {
      auto shard_of = [&](int tok) { return a.seq ? tok / a.n_loc : r; };
      auto row_in = [&](int tok) { return a.seq ? tok - (tok / a.n_loc) * a.n_loc : tok; };
      const int qx0 = a.seq ? r * a.Hl * D : 0, kx0 = a.seq ? (r * a.Hkvl + g) * D : g * D;
      if (!a.seq && lane == 0) {
        tma_prefetch_desc(&a.tq[r]);
        tma_prefetch_desc(&a.tdo[r]);
      }
      const CUtensorMap *mk = &a.tk[shard_of(n0)], *mv = &a.tv[shard_of(n0)];
      mbar_arrive_expect_tx_w(kv_full, 2 * L::kKV);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        tma_load_2d_w(sbase + L::kK + hf * (TB * 128), mk, kv_full, kx0 + hf * 64, row_in(n0));
        tma_load_2d_w(sbase + L::kV + hf * (TB * 128), mv, kv_full, kx0 + hf * 64, row_in(n0));
      }
      int it = 0;
      for (; it < T; ++it) {
        const int s = it % NST;
        if (!mbar_wait_warp(st_empty(s), ((it / NST) & 1) ^ 1, kErrBwd, 0x100 + s)) break;
        const int h = g * a.group + it / nrb;
        const int m0 = (rb_lo + it % nrb) * SB;
        const uint32_t stg = sbase + L::kRing + s * 2 * L::kBlk;
        mbar_arrive_expect_tx_w(st_full(s), 2 * L::kBlk + 512);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          tma_load_2d_w(stg + hf * (SB * 128), &a.tq[shard_of(m0)], st_full(s), qx0 + h * D + hf * 64, row_in(m0));
          tma_load_2d_w(stg + L::kBlk + hf * (SB * 128), &a.tdo[shard_of(m0)], st_full(s), qx0 + h * D + hf * 64,
                        row_in(m0));
        }
        const int64_t vo = (static_cast<int64_t>(r) * a.Hl + h) * a.Npad + m0;
        bulk_load_w(sbase + L::kVec + s * 512, a.lse2 + vo, SB * 4, st_full(s));
        bulk_load_w(sbase + L::kVec + s * 512 + 256, a.Dv + vo, SB * 4, st_full(s));
      }
      for (int k = it > NST ? it - NST : 0; k < it; ++k)
        mbar_wait_drain_w(st_full(k % NST), (k / NST) & 1, kErrBwd, 0x1f0);
      mbar_wait_drain_w(kv_full, 0, kErrBwd, 0x1f1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    {
      // Tensor-pipe order: S^T(i+1) dP^T(i+1) | dV(i) dK(i) | S^T(i+2) dP^T(i+2) | ...
      // S^T(i+2) reuses the columns dV(i) reads (P^T) and dP^T(i+2) the ones dK(i)
      // reads (dS^T): each waits only for its own reader, so one is always queued.
      constexpr uint32_t idS = idesc_bf16_f32(TB, SB, 0, 0);
      constexpr uint32_t idA = idesc_bf16_f32(TB, D, 0, 1);
      bool ok = mbar_wait_warp(kv_full, 0, kErrBwd, 0x200);
      tc_fence_after();
      auto stage = [&](int it) { return sbase + L::kRing + (it % NST) * 2 * L::kBlk; };
      // Descriptors built once; per MMA only a constant offset is added.
      const uint64_t dK0 = smem_desc_sw128(sbase + L::kK, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sbase + L::kV, 16, 1024);
      const uint64_t dRing0 = smem_desc_sw128(sbase + L::kRing, 16, 1024);
      const uint64_t dRingMN0 = smem_desc_sw128(sbase + L::kRing, SB * 128, 1024);
      auto issue_s = [&](int it) {
        const uint64_t qd = desc_adv(dRing0, (it % NST) * 2 * L::kBlk);
        const uint32_t dst = tS(it & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk / 4) * (TB * 128) + (kk % 4) * 32;
          const uint32_t qo = (kk / 4) * (SB * 128) + (kk % 4) * 32;
          mma_ss_w(dst, desc_adv(dK0, ko), desc_adv(qd, qo), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(s_full(it & 1));
      };
      auto issue_dp = [&](int it) {
        const uint64_t dod = desc_adv(dRing0, (it % NST) * 2 * L::kBlk + L::kBlk);
        const uint32_t dst = tDP(it & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk / 4) * (TB * 128) + (kk % 4) * 32;
          const uint32_t qo = (kk / 4) * (SB * 128) + (kk % 4) * 32;
          mma_ss_w(dst, desc_adv(dV0, ko), desc_adv(dod, qo), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(dp_full(it & 1));
      };
      // prologue: the first two streamed blocks
      for (int it = 0; it < 2 && it < T && ok; ++it) {
        if (!mbar_wait_warp(st_full(it % NST), (it / NST) & 1, kErrBwd, 0x210)) { ok = false; break; }
        tc_fence_after();
        issue_s(it);
        issue_dp(it);
      }
      for (int it = 0; it < T && ok; ++it) {
        const int b = it & 1;
        const uint32_t stg = stage(it);
        if (!mbar_wait_warp(p_full(b), (it >> 1) & 1, kErrBwd, 0x230)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dob = desc_adv(dRingMN0, stg - (sbase + L::kRing) + L::kBlk);
        const uint64_t qb = desc_adv(dRingMN0, stg - (sbase + L::kRing));
        const uint32_t aS = tS(b), aDP = tDP(b);
#pragma unroll
        for (int kk = 0; kk < SB / 16; ++kk)
          mma_ts_w(tDV, aS + kk * 8, desc_adv(dob, kk * 2048), idA, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit_w(dv_done(b));
        if (!mbar_wait_warp(ds_full(b), (it >> 1) & 1, kErrBwd, 0x240)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < SB / 16; ++kk)
          mma_ts_w(tDK, aDP + kk * 8, desc_adv(qb, kk * 2048), idA, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit_w(dk_done(b));
        mma_commit_w(st_empty(it % NST));
        const int nx = it + 2;
        if (nx < T) {
          if (!mbar_wait_warp(st_full(nx % NST), (nx / NST) & 1, kErrBwd, 0x210)) { ok = false; break; }
          if (!mbar_wait_warp(dv_done(b), (it >> 1) & 1, kErrBwd, 0x220)) { ok = false; break; }
          tc_fence_after();
          issue_s(nx);
          if (!mbar_wait_warp(dk_done(b), (it >> 1) & 1, kErrBwd, 0x221)) { ok = false; break; }
          tc_fence_after();
          issue_dp(nx);
        }
      }
      mma_commit_w(acc_done);
      mbar_wait_drain_w(acc_done, 0, kErrBwd, 0x250);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise
    const int b = warp >> 2;                            // this warpgroup's TMEM buffer
    const int lrow = 32 * (warp & 3) + lane;            // TMEM lane = key row
    const uint32_t loff = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int key = n0 + lrow;
    const int kde = doc_end_of(a.cu, a.num_seqs, min(key, N - 1), N);   // rows allowed: key <= row < kde
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int it = b; it < T; it += 2) {
      const int s = it % NST;
      const int m0 = (rb_lo + it % nrb) * SB;
      // lse*log2(e) and D of this block's 64 rows: same for every lane, read as
      // 16-byte shared-memory broadcasts
      const uint32_t vl = sbase + L::kVec + s * 512, vd = vl + 256;
      if (!mbar_wait_warp(st_full(s), (it / NST) & 1, kErrBwd, 0x300)) { ok = false; break; }
      if (!mbar_wait_warp(s_full(b), (it >> 1) & 1, kErrBwd, 0x310)) { ok = false; break; }
      tc_fence_after();
      uint32_t pv[SB];
      tmem_ld32(tS(b) + loff, *reinterpret_cast<uint32_t(*)[32]>(&pv[0]));
      tmem_ld32(tS(b) + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&pv[32]));
      tmem_wait_ld();
      const bool need_mask = (m0 < n0 + TB - 1) || (m0 + SB > doc_end_first);
      // allowed rows of this key within the block: c in [lo, hi)  <=>  (unsigned)(c - lo) < span
      const int lo = key - m0;
      const uint32_t span = static_cast<uint32_t>(max(kde - key, 0));
#pragma unroll
      for (int c = 0; c < SB; c += 4) {
        const float4 l4 = ld_shared_f4(vl + 4 * c);
        float p0 = ex2_approx(u2f(pv[c]) * sl2 - l4.x);
        float p1 = ex2_approx(u2f(pv[c + 1]) * sl2 - l4.y);
        float p2 = ex2_approx(u2f(pv[c + 2]) * sl2 - l4.z);
        float p3 = ex2_approx(u2f(pv[c + 3]) * sl2 - l4.w);
        if (need_mask) {
          p0 = static_cast<uint32_t>(c - lo) < span ? p0 : 0.f;
          p1 = static_cast<uint32_t>(c + 1 - lo) < span ? p1 : 0.f;
          p2 = static_cast<uint32_t>(c + 2 - lo) < span ? p2 : 0.f;
          p3 = static_cast<uint32_t>(c + 3 - lo) < span ? p3 : 0.f;
        }
        pv[c] = __float_as_uint(p0);
        pv[c + 1] = __float_as_uint(p1);
        pv[c + 2] = __float_as_uint(p2);
        pv[c + 3] = __float_as_uint(p3);
      }
      uint32_t pk[SB / 2];
#pragma unroll
      for (int c = 0; c < SB / 2; ++c) pk[c] = pack_bf16x2(u2f(pv[2 * c]), u2f(pv[2 * c + 1]));
      tmem_st32(tS(b) + loff, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(b));
      if (!mbar_wait_warp(dp_full(b), (it >> 1) & 1, kErrBwd, 0x320)) { ok = false; break; }
      tc_fence_after();
      uint32_t dp[SB];
      tmem_ld32(tDP(b) + loff, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_ld32(tDP(b) + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < SB; c += 4) {
        const float4 d4 = ld_shared_f4(vd + 4 * c);
        const float d0 = u2f(pv[c]) * (u2f(dp[c]) - d4.x);
        const float d1 = u2f(pv[c + 1]) * (u2f(dp[c + 1]) - d4.y);
        const float d2 = u2f(pv[c + 2]) * (u2f(dp[c + 2]) - d4.z);
        const float d3 = u2f(pv[c + 3]) * (u2f(dp[c + 3]) - d4.w);
        dp[c / 2] = pack_bf16x2(d0, d1);     // in place: dp[c/2], dp[c/2+1] are already consumed
        dp[c / 2 + 1] = pack_bf16x2(d2, d3);
      }
      tmem_st32(tDP(b) + loff, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full(b));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK
    if (ok && mbar_wait_warp(acc_done, 0, kErrBwd, 0x330)) {
      tc_fence_after();
      const uint32_t src = (b == 0 ? tDV : tDK) + loff;
      const float mul = b == 0 ? 1.f : a.scale;
      const int kb = a.seq ? min(key, N - 1) / a.n_loc : r;     // clamped: rows >= N are not stored
      const int64_t krow = a.seq ? (static_cast<int64_t>(key - kb * a.n_loc) * (a.Hkvl * a.P) + r * a.Hkvl + g)
                                 : (static_cast<int64_t>(key) * a.Hkvl + g);
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(b == 0 ? a.dv.p[kb] : a.dk.p[kb]) + krow * D;
#pragma unroll 1
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t v[32];
        tmem_ld32(src + c4 * 32, v);
        tmem_wait_ld();
        uint4 o4[4];
        uint32_t* ow = reinterpret_cast<uint32_t*>(o4);
#pragma unroll
        for (int e = 0; e < 16; ++e) ow[e] = pack_bf16x2(u2f(v[2 * e]) * mul, u2f(v[2 * e + 1]) * mul);
        if (key < N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c4 * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = o4[e];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ====================================================================== dQ
// One CTA per 128-row block of one query head. Q and dO stay in shared memory;
// 128-key blocks of K and V stream through two rings (K: 3 stages, V: 2), so
// every MMA is N=128 wide (half the shared-memory operand traffic per FLOP of
// 64-key blocks):
//   S = Q K^T (S double-buffered in TMEM), dP = dO V^T (single buffer),
//   dS = P (dP - D_i) elementwise: both warpgroups work on the same block, one
//   thread per row, warpgroup w on keys [64w, 64w+64); each writes its dS as
//   bf16 over the start of its own S columns, and dQ += dS K is issued as two
//   K=64 halves that read those two column ranges.
// Tensor-pipe order per block i: dP(i+1) | dQ(i) | S(i+2): dP(i+1) goes out as
// soon as the elementwise warps hold dP(i) in registers (a barrier of its own,
// before they start computing), so it runs under their arithmetic and they can
// start block i+1 as soon as they finish block i.
struct DqArgs {
  CUtensorMap tq[kMaxRanks];    // box 64 cols x TB rows
  CUtensorMap tdo[kMaxRanks];   // box 64 cols x TB rows
  CUtensorMap tk[kMaxRanks];    // box 64 cols x TB rows
  CUtensorMap tv[kMaxRanks];    // box 64 cols x TB rows
  RankPtrsMut dq;
  const float* lse2;
  const float* Dv;
  const int32_t* cu;
  int num_seqs;
  int N, Npad, Hl, Hkvl, group;
  float scale, scale_log2;
  int rank_lo;
  int num_m_tiles;
  int seq, n_loc, P;
};

constexpr int kNK = 3, kNV = 2;   // K and V ring depths in the dQ kernel

template <int D>
struct DqLayout {
  static constexpr uint32_t kTile = TB * D * 2;        // 128 rows (or keys) x D
  static constexpr uint32_t kQ = 0, kDO = kTile;
  static constexpr uint32_t kKRing = 2 * kTile;
  static constexpr uint32_t kVRing = kKRing + kNK * kTile;
  static constexpr uint32_t kBars = kVRing + kNV * kTile;
  // q_full, k_full[3], k_empty[3], v_full[2], v_empty[2], s_full[2], dp_full, ds_full, dq_done[2], acc_done,
  // dp_free
  static constexpr int kNumBars = 1 + 2 * kNK + 2 * kNV + 2 + 1 + 1 + 2 + 1 + 1;
  static constexpr uint32_t kSlot = kBars + kNumBars * 8;
  static constexpr uint32_t kAlloc = kSlot + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dq_kernel(const __grid_constant__ DqArgs a) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t bars = sbase + L::kBars;
  const uint32_t q_full = bars;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + kNK + s); };
  auto v_full = [&](int s) { return bars + 8u * (1 + 2 * kNK + s); };
  auto v_empty = [&](int s) { return bars + 8u * (1 + 2 * kNK + kNV + s); };
  auto s_full = [&](int b) { return bars + 8u * (1 + 2 * kNK + 2 * kNV + b); };
  const uint32_t dp_full = bars + 8u * (3 + 2 * kNK + 2 * kNV);
  const uint32_t ds_full = bars + 8u * (4 + 2 * kNK + 2 * kNV);
  auto dq_done = [&](int b) { return bars + 8u * (5 + 2 * kNK + 2 * kNV + b); };
  const uint32_t acc_done = bars + 8u * (7 + 2 * kNK + 2 * kNV);
  const uint32_t dp_free = bars + 8u * (8 + 2 * kNK + 2 * kNV);
  volatile uint32_t* slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x % a.Hl;
  const int r = a.rank_lo + blockIdx.x / a.Hl;
  const int g = h / a.group;
  const int N = a.N;
  const int m0 = (a.num_m_tiles - 1 - static_cast<int>(blockIdx.y)) * TB;   // longest first
  const int m_last = min(m0 + TB, N) - 1;
  const int kb_lo = doc_start_of(a.cu, a.num_seqs, m0) / TB;
  const int T = m_last / TB + 1 - kb_lo;
  const int max_start = doc_start_of(a.cu, a.num_seqs, m_last);

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bars + 8u * i, 1);
    mbar_init(ds_full, 256);
    mbar_init(dp_free, 256);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sbase + L::kSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t tDQ = tmem, tDP = tmem + 384u;
  auto tS = [&](int b) { return tmem + 128u + 128u * b; };

  if (warp == kTmaWarp) {
    {
      auto shard_of = [&](int tok) { return a.seq ? tok / a.n_loc : r; };
      auto row_in = [&](int tok) { return a.seq ? tok - (tok / a.n_loc) * a.n_loc : tok; };
      const int qx0 = a.seq ? (r * a.Hl + h) * D : h * D, kx0 = a.seq ? (r * a.Hkvl + g) * D : g * D;
      if (!a.seq && lane == 0) {
        tma_prefetch_desc(&a.tk[r]);
        tma_prefetch_desc(&a.tv[r]);
      }
      mbar_arrive_expect_tx_w(q_full, 2 * L::kTile);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        tma_load_2d_w(sbase + L::kQ + hf * (TB * 128), &a.tq[shard_of(m0)], q_full, qx0 + hf * 64, row_in(m0));
        tma_load_2d_w(sbase + L::kDO + hf * (TB * 128), &a.tdo[shard_of(m0)], q_full, qx0 + hf * 64, row_in(m0));
      }
      int nk = 0, nv = 0;     // blocks of K and of V issued
      for (int j = 0; j < T; ++j) {
        const int k0 = (kb_lo + j) * TB;
        const int ks = j % kNK, vs = j % kNV;
        if (!mbar_wait_warp(k_empty(ks), ((j / kNK) & 1) ^ 1, kErrBwd, 0x500 + ks)) break;
        mbar_arrive_expect_tx_w(k_full(ks), L::kTile);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_2d_w(sbase + L::kKRing + ks * L::kTile + hf * (TB * 128), &a.tk[shard_of(k0)], k_full(ks),
                        kx0 + hf * 64, row_in(k0));
        ++nk;
        if (!mbar_wait_warp(v_empty(vs), ((j / kNV) & 1) ^ 1, kErrBwd, 0x508 + vs)) break;
        mbar_arrive_expect_tx_w(v_full(vs), L::kTile);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_2d_w(sbase + L::kVRing + vs * L::kTile + hf * (TB * 128), &a.tv[shard_of(k0)], v_full(vs),
                        kx0 + hf * 64, row_in(k0));
        ++nv;
      }
      // Drain: every issued load must land before the CTA can exit.
      for (int k = nk > kNK ? nk - kNK : 0; k < nk; ++k)
        mbar_wait_drain_w(k_full(k % kNK), (k / kNK) & 1, kErrBwd, 0x5f0);
      for (int k = nv > kNV ? nv - kNV : 0; k < nv; ++k)
        mbar_wait_drain_w(v_full(k % kNV), (k / kNV) & 1, kErrBwd, 0x5f2);
      mbar_wait_drain_w(q_full, 0, kErrBwd, 0x5f1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    {
      constexpr uint32_t idS = idesc_bf16_f32(TB, TB, 0, 0);
      constexpr uint32_t idA = idesc_bf16_f32(TB, D, 0, 1);
      bool ok = mbar_wait_warp(q_full, 0, kErrBwd, 0x600);
      tc_fence_after();
      const uint64_t dQ0 = smem_desc_sw128(sbase + L::kQ, 16, 1024);
      const uint64_t dDO0 = smem_desc_sw128(sbase + L::kDO, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sbase + L::kKRing, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sbase + L::kVRing, 16, 1024);
      const uint64_t dKmn0 = smem_desc_sw128(sbase + L::kKRing, TB * 128, 1024);
      auto issue_s = [&](int it) -> bool {
        if (!mbar_wait_warp(k_full(it % kNK), (it / kNK) & 1, kErrBwd, 0x610)) return false;
        tc_fence_after();
        const uint64_t kd = desc_adv(dK0, (it % kNK) * L::kTile);
        const uint32_t dst = tS(it & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk / 4) * (TB * 128) + (kk % 4) * 32;
          mma_ss_w(dst, desc_adv(dQ0, o), desc_adv(kd, o), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(s_full(it & 1));
        return true;
      };
      auto issue_dp = [&](int it) -> bool {
        if (!mbar_wait_warp(v_full(it % kNV), (it / kNV) & 1, kErrBwd, 0x611)) return false;
        tc_fence_after();
        const uint64_t vd = desc_adv(dV0, (it % kNV) * L::kTile);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk / 4) * (TB * 128) + (kk % 4) * 32;
          mma_ss_w(tDP, desc_adv(dDO0, o), desc_adv(vd, o), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(dp_full);
        return true;
      };
      if (ok && T > 0) ok = issue_s(0) && issue_dp(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int it = 0; it < T && ok; ++it) {
        const int b = it & 1;
        if (!mbar_wait_warp(dp_free, it & 1, kErrBwd, 0x631)) { ok = false; break; }
        tc_fence_after();
        mma_commit_w(v_empty(it % kNV));                 // dP(it) has completed: V(it) is free
        if (it + 1 < T && !issue_dp(it + 1)) { ok = false; break; }
        if (!mbar_wait_warp(ds_full, it & 1, kErrBwd, 0x630)) { ok = false; break; }
        tc_fence_after();
        // dQ += dS K: keys [0,64) from S columns [0,32), keys [64,128) from [64,96)
        const uint64_t kmn = desc_adv(dKmn0, (it % kNK) * L::kTile);
#pragma unroll
        for (int kk = 0; kk < TB / 16; ++kk) {
          const uint32_t acol = (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8;
          mma_ts_w(tDQ, tS(b) + acol, desc_adv(kmn, kk * 2048), idA, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_w(dq_done(b));
        mma_commit_w(k_empty(it % kNK));
        if (it + 2 < T) {
          if (!mbar_wait_warp(dq_done(b), (it >> 1) & 1, kErrBwd, 0x620)) { ok = false; break; }
          tc_fence_after();
          if (!issue_s(it + 2)) { ok = false; break; }
        }
      }
      mma_commit_w(acc_done);
      mbar_wait_drain_w(acc_done, 0, kErrBwd, 0x640);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise
    const int wg = warp >> 2;                            // key half of every block
    const int lrow = 32 * (warp & 3) + lane;             // TMEM lane = query row
    const uint32_t loff = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int i = m0 + lrow;
    const int ic = min(i, N - 1);
    const int st_i = doc_start_of(a.cu, a.num_seqs, ic);
    const int64_t vo = (static_cast<int64_t>(r) * a.Hl + h) * a.Npad + i;   // padded: always in bounds
    const float lse2_i = a.lse2[vo];
    const float D_i = a.Dv[vo];
    const float sl2 = a.scale_log2;
    const uint32_t col0 = 64u * wg;
    bool ok = true;
    for (int it = 0; it < T; ++it) {
      const int k0 = (kb_lo + it) * TB + 64 * wg;
      const uint32_t sb = tS(it & 1) + col0 + loff;
      if (!mbar_wait_warp(s_full(it & 1), (it >> 1) & 1, kErrBwd, 0x700)) { ok = false; break; }
      tc_fence_after();
      uint32_t pv[64], dp[64];
      tmem_ld32(sb, *reinterpret_cast<uint32_t(*)[32]>(&pv[0]));
      tmem_ld32(sb + 32, *reinterpret_cast<uint32_t(*)[32]>(&pv[32]));
      if (!mbar_wait_warp(dp_full, it & 1, kErrBwd, 0x710)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32(tDP + col0 + loff, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_ld32(tDP + col0 + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(dp_free);                                // dP(it) is in registers: dP(it+1) may overwrite it
      const bool need_mask = (k0 + 63 > m0) || (k0 < max_start);
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float p0 = ex2_approx(u2f(pv[c]) * sl2 - lse2_i);
        float p1 = ex2_approx(u2f(pv[c + 1]) * sl2 - lse2_i);
        if (need_mask) {
          const int key = k0 + c;
          if (key > i || key < st_i) p0 = 0.f;
          if (key + 1 > i || key + 1 < st_i) p1 = 0.f;
        }
        pv[c / 2] = pack_bf16x2(p0 * (u2f(dp[c]) - D_i), p1 * (u2f(dp[c + 1]) - D_i));   // in place
      }
      tmem_st32(sb, *reinterpret_cast<uint32_t(*)[32]>(&pv[0]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // epilogue: each warpgroup writes half of the dQ row (columns wg*D/2 ...)
    if (ok && mbar_wait_warp(acc_done, 0, kErrBwd, 0x720)) {
      tc_fence_after();
      const int qb = a.seq ? ic / a.n_loc : r;           // ic clamped: rows >= N are not stored
      const int64_t qrow = a.seq ? (static_cast<int64_t>(ic - qb * a.n_loc) * (a.Hl * a.P) + r * a.Hl + h)
                                 : (static_cast<int64_t>(i) * a.Hl + h);
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.dq.p[qb]) + qrow * D;
#pragma unroll 1
      for (int c4 = wg * (D / 64); c4 < (wg + 1) * (D / 64); ++c4) {
        uint32_t v[32];
        tmem_ld32(tDQ + loff + c4 * 32, v);
        tmem_wait_ld();
        uint4 o4[4];
        uint32_t* ow = reinterpret_cast<uint32_t*>(o4);
#pragma unroll
        for (int e = 0; e < 16; ++e) ow[e] = pack_bf16x2(u2f(v[2 * e]) * a.scale, u2f(v[2 * e + 1]) * a.scale);
        if (i < N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c4 * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = o4[e];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd_sm100
}  // namespace uly

#include "attn_bwd_onepass_sm100.cuh"

namespace uly {
namespace bwd_sm100 {

// ====================================================================== host
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool encode(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t rows, int64_t row_elems, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_elems), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_elems * 2)};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int padded_rows(int N) { return (N + TB - 1) / TB * TB; }

template <int D>
cudaError_t launch_all(const AttnShape& s, const PrepArgs& pa, const DkdvArgs& ka, const DqArgs& qa,
                       cudaStream_t stream) {
  const int nranks = s.rank_hi - s.rank_lo;
  {
    constexpr int RPB = 256 / (D / 8);
    const int64_t rows = static_cast<int64_t>(pa.Npad) * s.Hl * nranks;
    bwd_prep_kernel<D><<<static_cast<unsigned>((rows + RPB - 1) / RPB), 256, 0, stream>>>(pa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DkdvLayout<D>::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid(s.Hkvl * nranks, (s.N + TB - 1) / TB);
    attn_bwd_dkdv_kernel<D><<<grid, kThreads, DkdvLayout<D>::kAlloc, stream>>>(ka);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DqLayout<D>::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid(s.Hl * nranks, qa.num_m_tiles);
    attn_bwd_dq_kernel<D><<<grid, kThreads, DqLayout<D>::kAlloc, stream>>>(qa);
    return cudaGetLastError();
  }
}

// prep, zero the dQ accumulator of the ranks in range, one-pass dK/dV/dQ, dQ conversion
cudaError_t launch_onepass(const AttnShape& s, const PrepArgs& pa, const DkdvArgs& ka, const RankPtrsMut& dq,
                           cudaStream_t stream) {
  constexpr int D = onepass::D;
  const int nranks = s.rank_hi - s.rank_lo;
  {
    constexpr int RPB = 256 / (D / 8);
    const int64_t rows = static_cast<int64_t>(pa.Npad) * s.Hl * nranks;
    bwd_prep_kernel<D><<<static_cast<unsigned>((rows + RPB - 1) / RPB), 256, 0, stream>>>(pa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t per_rank = static_cast<size_t>(s.Hl) * pa.Npad * D;   // floats
  {
    cudaError_t e = cudaMemsetAsync(ka.dqacc + per_rank * s.rank_lo, 0, per_rank * nranks * sizeof(float), stream);
    if (e != cudaSuccess) return e;
  }
  {
    cudaError_t e = cudaFuncSetAttribute(onepass::attn_bwd_onepass_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, onepass::Layout::kAlloc);
    if (e != cudaSuccess) return e;
    const int nkb = (s.N + TB - 1) / TB;
    dim3 grid = ka.kb_fast ? dim3(nkb, s.Hkvl * nranks) : dim3(s.Hkvl * nranks, nkb);
    onepass::attn_bwd_onepass_kernel<<<grid, onepass::kOpThreads, onepass::Layout::kAlloc, stream>>>(ka);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    onepass::ConvArgs ca;
    memset(&ca, 0, sizeof(ca));
    ca.acc = ka.dqacc;
    ca.dq = dq;
    ca.N = s.N;
    ca.Npad = pa.Npad;
    ca.Hl = s.Hl;
    ca.rank_lo = s.rank_lo;
    ca.nranks = nranks;
    ca.scale = s.scale;
    ca.seq = pa.seq;
    ca.n_loc = pa.n_loc;
    ca.P = s.P;
    const int64_t threads = static_cast<int64_t>(nranks) * s.Hl * (pa.Npad / 4) * 32;
    onepass::dq_convert_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(ca);
    return cudaGetLastError();
  }
}

}  // namespace bwd_sm100

bool attn_bwd_onepass(int d, int deterministic) { return !deterministic && d == bwd_sm100::onepass::D; }

// The one-pass kernel uses all but a few hundred bytes of a CTA's shared memory
// and aligns its tiles to 1024 bytes, so it fits only when its dynamic shared
// memory starts close enough below a 1024-byte boundary. The dynamic area
// starts after the per-block reserved shared memory and the kernel's static
// shared memory: given that offset, does the layout fit?
bool attn_bwd_onepass_layout_fits(uint32_t dyn_base_offset) {
  const uint32_t pad = (1024u - dyn_base_offset % 1024u) % 1024u;
  return pad + bwd_sm100::onepass::Layout::kUsed <= bwd_sm100::onepass::Layout::kAlloc;
}

// Whether the one-pass kernel's layout fits on the current device (looked up
// once per device). When it does not, the backward runs the two-pass kernels
// instead of returning an error: same dK/dV bits, dQ to summation order.
bool attn_bwd_onepass_usable() {
  constexpr int kMaxDev = 64;
  static int cache[kMaxDev] = {};   // 0 unknown, 1 fits, 2 does not
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  if (cache[dev] == 0) {
    int reserved = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, bwd_sm100::onepass::attn_bwd_onepass_kernel) != cudaSuccess)
      return false;
    cache[dev] = attn_bwd_onepass_layout_fits(static_cast<uint32_t>(reserved + fa.sharedSizeBytes)) ? 1 : 2;
  }
  return cache[dev] == 1;
}

size_t attn_bwd_seq_workspace_bytes(int64_t N, int P, int Hl, int d, int deterministic) {
  size_t bytes = attn_bwd_workspace_bytes(N, P, Hl, d, deterministic);
  if (attn_bwd_onepass(d, deterministic)) bytes += 2 * static_cast<size_t>(P) * N * Hl * d * 2;
  return bytes;
}

size_t attn_bwd_workspace_bytes(int64_t N, int P, int Hl, int d, int deterministic) {
  const int64_t npad = (N + bwd_sm100::TB - 1) / bwd_sm100::TB * bwd_sm100::TB;
  size_t bytes = 2 * static_cast<size_t>(P) * Hl * npad * sizeof(float);
  if (attn_bwd_onepass(d, deterministic)) bytes += static_cast<size_t>(P) * Hl * npad * d * sizeof(float);
  return bytes;
}

namespace bwd_sm100 {
// Streaming multiprocessors of the current device (looked up once per device;
// 148 on B200 if the query fails).
int device_sm_count() {
  constexpr int kMaxDev = 64;
  static int cache[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cache[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
  }
  return cache[dev];
}

// Fills everything but the per-buffer pointers and tensor maps, then launches.
// qdo_head (seq == 1 only): qa.tq / qa.tdo map head-sharded copies of Q and dO
// instead of the sequence shards.
cudaError_t launch_common(const AttnShape& s, PrepArgs& pa, DkdvArgs& ka, DqArgs& qa, void* workspace, int seq,
                          int deterministic, cudaStream_t stream, bool qdo_head = false) {
  const int Npad = padded_rows(s.N);
  float* lse2 = static_cast<float*>(workspace);
  float* Dv = lse2 + static_cast<size_t>(s.P) * s.Hl * Npad;
  pa.lse2 = lse2;
  pa.Dv = Dv;
  pa.N = s.N;
  pa.Npad = Npad;
  pa.Hl = s.Hl;
  pa.rank_lo = s.rank_lo;
  pa.nranks = s.rank_hi - s.rank_lo;
  pa.seq = ka.seq = qa.seq = seq;
  ka.qdo_seq = seq && !qdo_head ? 1 : 0;
  pa.n_loc = ka.n_loc = qa.n_loc = s.N / s.P;
  pa.P = ka.P = qa.P = s.P;
  ka.lse2 = qa.lse2 = lse2;
  ka.Dv = qa.Dv = Dv;
  ka.cu = qa.cu = s.cu_seqlens;
  ka.num_seqs = qa.num_seqs = s.num_seqs;
  ka.N = qa.N = s.N;
  ka.Npad = qa.Npad = Npad;
  ka.Hl = qa.Hl = s.Hl;
  ka.Hkvl = qa.Hkvl = s.Hkvl;
  ka.group = qa.group = s.Hl / s.Hkvl;
  ka.scale = qa.scale = s.scale;
  ka.scale_log2 = qa.scale_log2 = s.scale * kLog2e;
  ka.rank_lo = qa.rank_lo = s.rank_lo;
  qa.num_m_tiles = (s.N + TB - 1) / TB;
  if (attn_bwd_onepass(s.d, deterministic) && attn_bwd_onepass_usable()) {
    ka.dqacc = Dv + static_cast<size_t>(s.P) * s.Hl * Npad;   // 512-byte aligned: Npad is a multiple of 128
    // the one-pass kernel streams 128-row Q and dO blocks: the dQ kernel's maps
    memcpy(ka.tq, qa.tq, sizeof(ka.tq));
    memcpy(ka.tdo, qa.tdo, sizeof(ka.tdo));
    // Launch order. With the key block as the fast grid index, the CTAs
    // resident together serve one (rank, kv head) and keep its Q/dO blocks
    // and accumulator rows in L2 (DRAM traffic 3.8 instead of 8.5 GB per call
    // at varlen 64K). But a pair's heaviest CTAs (its first key blocks, which
    // stream the most query blocks) then start wherever the pair comes in the
    // grid, the last pair's near the end, and with few key blocks per pair
    // they form a long tail (8K tokens: 793 against 936 TFLOP/s). So the key
    // block leads only when each pair has at least two waves' worth of key
    // blocks; otherwise the kv head does and every pair's heaviest blocks
    // start first.
    ka.kb_fast = (s.N + TB - 1) / TB >= 2 * device_sm_count() ? 1 : 0;
    return launch_onepass(s, pa, ka, qa.dq, stream);
  }
  return s.d == 64 ? launch_all<64>(s, pa, ka, qa, stream) : launch_all<128>(s, pa, ka, qa, stream);
}
}  // namespace bwd_sm100

cudaError_t launch_attn_bwd(const AttnShape& s, const void* const* q, const void* const* k, const void* const* v,
                            const void* const* o, const float* const* lse, const void* const* dO, void* const* dq,
                            void* const* dk, void* const* dv, void* workspace, int deterministic,
                            cudaStream_t stream) {
  using namespace bwd_sm100;
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return cudaErrorNotSupported;
  PrepArgs pa;
  memset(&pa, 0, sizeof(pa));
  DkdvArgs ka;
  memset(&ka, 0, sizeof(ka));
  DqArgs qa;
  memset(&qa, 0, sizeof(qa));
  const int64_t qe = static_cast<int64_t>(s.Hl) * s.d, ke = static_cast<int64_t>(s.Hkvl) * s.d;
  for (int r = s.rank_lo; r < s.rank_hi; ++r) {
    pa.o.p[r] = o[r];
    pa.dO.p[r] = dO[r];
    pa.lse.p[r] = lse[r];
    if (!encode(enc, &ka.tq[r], q[r], s.N, qe, SB) || !encode(enc, &ka.tdo[r], dO[r], s.N, qe, SB) ||
        !encode(enc, &ka.tk[r], k[r], s.N, ke, TB) || !encode(enc, &ka.tv[r], v[r], s.N, ke, TB) ||
        !encode(enc, &qa.tq[r], q[r], s.N, qe, TB) || !encode(enc, &qa.tdo[r], dO[r], s.N, qe, TB) ||
        !encode(enc, &qa.tk[r], k[r], s.N, ke, TB) || !encode(enc, &qa.tv[r], v[r], s.N, ke, TB))
      return cudaErrorInvalidValue;
    ka.dk.p[r] = dk[r];
    ka.dv.p[r] = dv[r];
    qa.dq.p[r] = dq[r];
  }
  return launch_common(s, pa, ka, qa, workspace, 0, deterministic, stream);
}

cudaError_t launch_attn_bwd_seq(const AttnShape& s, const void* const* q_seq, const void* const* k_seq,
                                const void* const* v_seq, const void* const* o_seq, const float* const* lse,
                                const void* const* do_seq, void* const* dq_seq, void* const* dk_seq,
                                void* const* dv_seq, void* workspace, size_t workspace_bytes, int deterministic,
                                cudaStream_t stream) {
  using namespace bwd_sm100;
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return cudaErrorNotSupported;
  PrepArgs pa;
  memset(&pa, 0, sizeof(pa));
  DkdvArgs ka;
  memset(&ka, 0, sizeof(ka));
  DqArgs qa;
  memset(&qa, 0, sizeof(qa));
  const int64_t n = s.N / s.P;
  const int64_t qe = static_cast<int64_t>(s.Hl) * s.P * s.d, ke = static_cast<int64_t>(s.Hkvl) * s.P * s.d;
  for (int p = 0; p < s.P; ++p) {
    pa.o.p[p] = o_seq[p];
    pa.dO.p[p] = do_seq[p];
    if (!encode(enc, &ka.tq[p], q_seq[p], n, qe, SB) || !encode(enc, &ka.tdo[p], do_seq[p], n, qe, SB) ||
        !encode(enc, &ka.tk[p], k_seq[p], n, ke, TB) || !encode(enc, &ka.tv[p], v_seq[p], n, ke, TB) ||
        !encode(enc, &qa.tq[p], q_seq[p], n, qe, TB) || !encode(enc, &qa.tdo[p], do_seq[p], n, qe, TB) ||
        !encode(enc, &qa.tk[p], k_seq[p], n, ke, TB) || !encode(enc, &qa.tv[p], v_seq[p], n, ke, TB))
      return cudaErrorInvalidValue;
    ka.dk.p[p] = dk_seq[p];
    ka.dv.p[p] = dv_seq[p];
    qa.dq.p[p] = dq_seq[p];
  }
  for (int r = s.rank_lo; r < s.rank_hi; ++r) pa.lse.p[r] = lse[r];
  // One-pass mode with room in the workspace: stage Q and dO in head shards
  // (one permute launch each) and let the kernel stream them from there; it
  // reads 128-row blocks whose rows are (H/P)*d*2 bytes apart instead of
  // H*d*2 in the sequence shards, which the TMA serves faster.
  bool qdo_head = false;
  if (attn_bwd_onepass(s.d, deterministic) && attn_bwd_onepass_usable() &&
      workspace_bytes >= attn_bwd_seq_workspace_bytes(s.N, s.P, s.Hl, s.d, deterministic)) {
    const size_t shard = static_cast<size_t>(s.N) * s.Hl * s.d * 2;
    char* base = static_cast<char*>(workspace) + attn_bwd_workspace_bytes(s.N, s.P, s.Hl, s.d, deterministic);
    void* qh[kMaxRanks] = {};
    void* doh[kMaxRanks] = {};
    for (int r = s.rank_lo; r < s.rank_hi; ++r) {
      qh[r] = base + static_cast<size_t>(r) * shard;
      doh[r] = base + static_cast<size_t>(s.P + r) * shard;
    }
    const int hx[3] = {s.Hl * s.P, s.Hkvl * s.P, s.Hkvl * s.P};
    const void* const* src_q[3] = {q_seq, nullptr, nullptr};
    void* const* dst_q[3] = {qh, nullptr, nullptr};
    const void* const* src_do[3] = {do_seq, nullptr, nullptr};
    void* const* dst_do[3] = {doh, nullptr, nullptr};
    cudaError_t e = launch_permute(true, src_q, dst_q, hx, s.N, s.P, s.d, s.rank_lo, s.rank_hi, stream);
    if (e == cudaSuccess) e = launch_permute(true, src_do, dst_do, hx, s.N, s.P, s.d, s.rank_lo, s.rank_hi, stream);
    if (e != cudaSuccess) return e;
    const int64_t qeh = static_cast<int64_t>(s.Hl) * s.d;
    for (int r = s.rank_lo; r < s.rank_hi; ++r)
      if (!encode(enc, &qa.tq[r], qh[r], s.N, qeh, TB) || !encode(enc, &qa.tdo[r], doh[r], s.N, qeh, TB))
        return cudaErrorInvalidValue;
    qdo_head = true;
  }
  return launch_common(s, pa, ka, qa, workspace, 1, deterministic, stream, qdo_head);
}

}  // namespace uly
