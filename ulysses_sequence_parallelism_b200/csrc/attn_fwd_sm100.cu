// Causal GQA (packed-varlen) flash-attention forward for sm_100a: tcgen05 MMA
// with TMEM accumulators, TMA-fed shared-memory tiles, warp-specialised.
//
// Computes, per rank in range, per local query head h, per row i:
//   s_ij = scale * q_i.k_j  (j <= i, same document),  o_i = softmax_j(s_i) V,
//   lse_i = ln sum_j exp(s_ij)
// (each rank runs attention by itself on its own heads over the whole
// sequence, the heads not interacting -- theaicatchup.com, "How Does Ulysses
// Sequence Parallelism Actually Work?").
//
// One CTA owns two 128-row query tiles of one head (256 rows) and streams the
// 128-key K/V blocks they need through a 4-stage shared-memory ring:
//   warp 8      : TMA producer (Q tiles once, then K_j, V_j alternately)
//   warp 9      : MMA issuer: S_t = Q_t K_j^T (SS, K-major both, N = 128),
//                 then O_t += P_t V_j (A = P from TMEM, B = V MN-major)
//   warps 0-3/4-7: softmax of tile 0 / tile 1, one thread per row: reads its
//                 S row from TMEM, online softmax in the log2 domain with fp32
//                 statistics, writes P (bf16) back over S, rescales its O row
//                 in TMEM only when its running max grew by more than 2^8
//                 (the result is exact either way: O and l share the max),
//                 and finally normalises O and stores O and LSE.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// Every wait on an mbarrier is bounded; a wait that runs out records an error
// in the library's device error word and the CTA drains and exits.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace uly {
namespace fwd_sm100 {

using namespace sm100;

constexpr int BM = 128;        // query rows per tile (two tiles per CTA)
constexpr int BN = 128;        // keys per K/V block
constexpr int NSTAGE = 4;      // K/V ring stages (K and V blocks alternate)
// Three warpgroups: two softmax warpgroups (warps 0-3, 4-7) and one holding
// the TMA producer (warp 8), the MMA issuer (warp 9) and two idle warps. At
// launch every thread gets 168 registers (3 warps per SM sub-partition share
// its 16K registers); the TMA/MMA warpgroup then gives registers back
// (setmaxnreg.dec to kRegsCtl) and the softmax warpgroups take them
// (setmaxnreg.inc to kRegsSoftmax): 2*128*208 + 128*88 = 384*168, exactly the
// launch's total, so every increase is covered.
constexpr int kThreads = 384;
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr int kRegsSoftmax = 208, kRegsCtl = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsCtl <= kThreads * 168, "register split above the launch total");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O when the max grows by > 2^8

// Two source/destination layouts share the kernel:
//  head layout (seq == 0): tq/tk/tv[r] map rank r's head shard [N, Hl*d]; o.p[r]
//    is rank r's head-sharded O.
//  sequence layout (seq == 1, the fused path): tq/tk/tv[p] map sequence shard p
//    [n, H*d] (n = N/P, a multiple of 128, so no 128-token tile straddles two
//    shards) and rank r's heads are the column slice starting at r*Hl*d;
//    o.p[p] is sequence shard p of O. The all-to-alls disappear into the
//    addressing: each tile is fetched from, and stored to, where it lives.
struct FwdArgs {
  CUtensorMap tq[kMaxRanks];
  CUtensorMap tk[kMaxRanks];
  CUtensorMap tv[kMaxRanks];
  RankPtrsMut o;
  RankPtrsF lse;
  const int32_t* cu;
  int num_seqs;
  int N, Hl, Hkvl, group;
  float scale_log2;
  int rank_lo;
  int num_m_blocks;   // blocks of 2*BM rows
  int seq;            // 1: sequence layout (see above)
  int n_loc;          // N / P
  int P;
};

template <int D>
struct Layout {
  static constexpr uint32_t kQTile = BM * D * 2;       // bytes of one Q tile
  static constexpr uint32_t kKV = BN * D * 2;          // bytes of one K or V block
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kRing = kQ + 2 * kQTile;
  static constexpr uint32_t kBars = kRing + NSTAGE * kKV;
  // barriers: q_full[2], kv_full[NS], kv_empty[NS], s_full[2], p_full[2], pv_done[2], mma_done
  static constexpr int kNumBars = 2 + 2 * NSTAGE + 2 + 2 + 2 + 1;
  static constexpr uint32_t kTmemSlot = kBars + kNumBars * 8;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;    // slack for 1024-byte alignment
};

ULY_DEV float u2f(uint32_t x) { return __uint_as_float(x); }

ULY_DEV float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_sm100_kernel(const __grid_constant__ FwdArgs a) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t sQ = sbase + L::kQ, sRing = sbase + L::kRing, bars = sbase + L::kBars;
  auto q_full = [&](int t) { return bars + 8u * t; };
  auto kv_full = [&](int s) { return bars + 8u * (2 + s); };
  auto kv_empty = [&](int s) { return bars + 8u * (2 + NSTAGE + s); };
  auto s_full = [&](int t) { return bars + 8u * (2 + 2 * NSTAGE + t); };
  auto p_full = [&](int t) { return bars + 8u * (4 + 2 * NSTAGE + t); };
  auto pv_done = [&](int t) { return bars + 8u * (6 + 2 * NSTAGE + t); };
  const uint32_t mma_done = bars + 8u * (8 + 2 * NSTAGE);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x % a.Hl;
  const int r = a.rank_lo + blockIdx.x / a.Hl;
  const int g = h / a.group;
  const int N = a.N;
  const int m0 = (a.num_m_blocks - 1 - static_cast<int>(blockIdx.y)) * (2 * BM);   // longest first

  // Per-tile row and key-block ranges (identical in every thread).
  bool active[2];
  int jb_begin[2], jb_end[2], first_row[2], last_row[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    first_row[t] = m0 + t * BM;
    last_row[t] = min(first_row[t] + BM, N) - 1;
    active[t] = first_row[t] < N;
    if (active[t]) {
      jb_begin[t] = doc_start_of(a.cu, a.num_seqs, first_row[t]) / BN;
      jb_end[t] = last_row[t] / BN + 1;
    } else {
      jb_begin[t] = jb_end[t] = 0;
    }
  }
  const int jb_lo = jb_begin[0];
  const int jb_hi = active[1] ? max(jb_end[0], jb_end[1]) : jb_end[0];

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bars + 8u * i, 1);
    mbar_init(p_full(0), 128);
    mbar_init(p_full(1), 128);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sbase + L::kTmemSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS[2] = {tmem, tmem + 128};
  const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};

  // Each role's code must sit inside the branch that changes its register
  // count (the compiler applies the new limit to the code the change dominates).
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    {
      // Map and coordinates of a token range: its shard and row within it.
      const int qx0 = a.seq ? (r * a.Hl + h) * D : h * D;
      const int kx0 = a.seq ? (r * a.Hkvl + g) * D : g * D;
      auto shard_of = [&](int tok) { return a.seq ? tok / a.n_loc : r; };
      auto row_in = [&](int tok) { return a.seq ? tok - (tok / a.n_loc) * a.n_loc : tok; };
      if (!a.seq && lane == 0) {
        tma_prefetch_desc(&a.tq[r]);
        tma_prefetch_desc(&a.tk[r]);
        tma_prefetch_desc(&a.tv[r]);
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!active[t]) continue;
        mbar_arrive_expect_tx_w(q_full(t), L::kQTile);
        const CUtensorMap* mq = &a.tq[shard_of(first_row[t])];
        const int qy = row_in(first_row[t]);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_2d_w(sQ + t * L::kQTile + hf * (BM * 128), mq, q_full(t), qx0 + hf * 64, qy);
      }
      uint32_t it = 0;
      bool ok = true;
      for (int jb = jb_lo; jb < jb_hi && ok; ++jb) {
        const int kp = shard_of(jb * BN), ky = row_in(jb * BN);
#pragma unroll
        for (int kind = 0; kind < 2; ++kind, ++it) {
          const int s = it % NSTAGE;
          const uint32_t ph = (it / NSTAGE) & 1u;
          if (!mbar_wait_warp(kv_empty(s), ph ^ 1u, kErrFwd, 0x100 + s)) { ok = false; break; }
          mbar_arrive_expect_tx_w(kv_full(s), L::kKV);
          const CUtensorMap* m = kind == 0 ? &a.tk[kp] : &a.tv[kp];
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_2d_w(sRing + s * L::kKV + hf * (BN * 128), m, kv_full(s), kx0 + hf * 64, ky);
        }
      }
      // Drain: every issued load must land before the CTA can exit.
      const uint32_t issued = it;
      for (uint32_t k = issued > NSTAGE ? issued - NSTAGE : 0; k < issued; ++k)
        mbar_wait_drain_w(kv_full(k % NSTAGE), (k / NSTAGE) & 1u, kErrFwd, 0x200);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (active[t]) mbar_wait_drain_w(q_full(t), 0, kErrFwd, 0x210 + t);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Order per key block j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1). P lives in
    // S's columns [0, 64), so S(j+1) is issued once PV(j) has read P. One
    // warp serves both tiles in this fixed order, which keeps the two tiles'
    // softmax phases alternating instead of competing for the exponential
    // unit (one issuing warp per tile measured 9 % slower).
    {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(BM, D, 0, 1);
      bool ok = true;
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (active[t] && !mbar_wait_warp(q_full(t), 0, kErrFwd, 0x300 + t)) ok = false;
      auto part = [&](int t, int jb) { return active[t] && jb >= jb_begin[t] && jb < jb_end[t]; };
      // Descriptors built once; per MMA only a constant offset is added.
      const uint64_t dQ0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dRing0 = smem_desc_sw128(sRing, 16, 1024);
      const uint64_t dRingV0 = smem_desc_sw128(sRing, BN * 128, 1024);
      // S_t = Q_t K^T over the whole 128-key block: N = 128 SS MMAs run at the
      // full tensor rate (two N = 64 halves are shared-memory bound, 48 cycles
      // per MMA instead of 32 per 64 columns).
      auto issue_s = [&](int t, uint32_t kb) {
        const uint64_t qd = desc_adv(dQ0, t * L::kQTile);
        const uint64_t kd = desc_adv(dRing0, kb - sRing);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_q = (kk / 4) * (BM * 128) + (kk % 4) * 32;
          const uint32_t off_k = (kk / 4) * (BN * 128) + (kk % 4) * 32;
          mma_ss_w(tS[t], desc_adv(qd, off_q), desc_adv(kd, off_k), idS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, uint32_t vb, int cnt) {
        const uint64_t vd = desc_adv(dRingV0, vb - sRing);
        const uint32_t a0 = tS[t], dst = tO[t];
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts_w(dst, a0 + kk * 8, desc_adv(vd, kk * (16 * 128)), idO, (cnt > 0 || kk > 0) ? 1u : 0u);
      };
      int cnt[2] = {0, 0};
      // prologue: S for the first key block (ring slot 0)
      if (ok && jb_lo < jb_hi) {
        if (!mbar_wait_warp(kv_full(0), 0, kErrFwd, 0x310)) {
          ok = false;
        } else {
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!part(t, jb_lo)) continue;
            issue_s(t, sRing);
            mma_commit_w(s_full(t));
          }
          mma_commit_w(kv_empty(0));
        }
      }
      for (int jb = jb_lo; jb < jb_hi && ok; ++jb) {
        const uint32_t itV = 2u * (jb - jb_lo) + 1u, itK = itV + 1u;
        const bool has_next = jb + 1 < jb_hi;
        if (!mbar_wait_warp(kv_full(itV % NSTAGE), (itV / NSTAGE) & 1u, kErrFwd, 0x330)) { ok = false; break; }
        if (has_next && !mbar_wait_warp(kv_full(itK % NSTAGE), (itK / NSTAGE) & 1u, kErrFwd, 0x311)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t vb = sRing + (itV % NSTAGE) * L::kKV;
        const uint32_t kb = sRing + (itK % NSTAGE) * L::kKV;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const bool now = part(t, jb), nxt = has_next && part(t, jb + 1);
          if (now) {
            if (!mbar_wait_warp(p_full(t), cnt[t] & 1, kErrFwd, 0x340 + t)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, vb, cnt[t]);
            mma_commit_w(pv_done(t));
            if (nxt) {
              // S(j+1) overwrites the columns P(j) is read from: after PV(j)
              if (!mbar_wait_warp(pv_done(t), cnt[t] & 1, kErrFwd, 0x320 + t)) { ok = false; break; }
              tc_fence_after();
              issue_s(t, kb);
              mma_commit_w(s_full(t));
            }
            ++cnt[t];
          } else if (nxt) {
            issue_s(t, kb);
            mma_commit_w(s_full(t));
          }
        }
        if (!ok) break;
        mma_commit_w(kv_empty(itV % NSTAGE));
        if (has_next) mma_commit_w(kv_empty(itK % NSTAGE));
      }
      // Drain: wait for every MMA issued above before TMEM can be released.
      mma_commit_w(mma_done);
      mbar_wait_drain_w(mma_done, 0, kErrFwd, 0x350);
    }
    __syncwarp();
  }   // warps 10 and 11: nothing to do
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax / epilogue
    // Per-warp scalars (no runtime-indexed arrays: they would live in local memory).
    const int t = warp >> 2;
    const int lrow = 32 * (warp & 3) + lane;        // TMEM lane = row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int frow = m0 + t * BM;
    const int lrow_t = min(frow + BM, N) - 1;
    const uint32_t tSt = tmem + 128u * t, tOt = tmem + 256u + D * t;
    if (frow < N) {
      const int i = frow + lrow;
      const bool row_ok = i < N;
      const int st_i = doc_start_of(a.cu, a.num_seqs, min(i, N - 1));
      const int max_start = doc_start_of(a.cu, a.num_seqs, lrow_t);
      const int jbb = doc_start_of(a.cu, a.num_seqs, frow) / BN, jbe = lrow_t / BN + 1;
      const float sl2 = a.scale_log2;
      float m_run = -INFINITY, l_run = 0.f;
      int cnt = 0;
      bool ok = true;
      for (int jb = jbb; jb < jbe; ++jb, ++cnt) {
        if (!mbar_wait_warp(s_full(t), cnt & 1, kErrFwd, 0x400 + t)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[BN];
        tmem_ld128(tSt + lane_off, v);
        tmem_wait_ld();
        const int n0 = jb * BN;
        const bool need_mask = (n0 + BN - 1 > frow) || (n0 < max_start);
        // Row max on the raw scores (the scale is positive, so it commutes with
        // max); masked keys become -inf and give exactly 0 below.
        if (need_mask) {
          const int lo = st_i - n0, hi = i - n0;   // allowed columns: lo <= c <= hi
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c < lo || c > hi) v[c] = __float_as_uint(-INFINITY);
        }
        float mx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = max3f(u2f(v[2 * e]), u2f(v[2 * e + 1]), -INFINITY);
#pragma unroll
        for (int c = 16; c < BN; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e) mx[e] = max3f(mx[e], u2f(v[c + 2 * e]), u2f(v[c + 2 * e + 1]));
        const float mraw = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        const float m_blk = mraw * sl2;           // -inf stays -inf
        const float m_new = fmaxf(m_run, m_blk);
        // Rescale decision (warp-uniform: TMEM loads/stores are warp-collective).
        bool rescale = false;
        float alpha = 1.f;
        if (cnt == 0) {
          m_run = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m_run + kRescaleThreshold)) {
          rescale = true;
          alpha = (m_new > m_run) ? ex2_approx(m_run - m_new) : 1.f;
          l_run *= alpha;
          m_run = m_new;
        }
        // p = 2^(s * scale*log2(e) - base): scale and subtraction in one packed
        // FFMA per two keys, then one ex2 each; row sum with packed adds.
        const float nbase = (m_run == -INFINITY) ? 0.f : -m_run;
        float rs[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) rs[e] = 0.f;
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          float x0, x1;
          ffma2_sc(x0, x1, u2f(v[c]), u2f(v[c + 1]), sl2, nbase);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          const int e = (c >> 1) & 3;
          fadd2_acc(rs[2 * e], rs[2 * e + 1], p0, p1);
          v[c / 2] = pack_bf16x2(p0, p1);
        }
        l_run += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
        tmem_st32(tSt + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_st32(tSt + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        if (rescale) {
          // O still holds the sum over earlier blocks at the old max: scale it
          // once the previous P.V has landed, before this block's P.V is issued.
          if (!mbar_wait_warp(pv_done(t), (cnt - 1) & 1, kErrFwd, 0x410 + t)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t ov[32];
            tmem_ld32(tOt + lane_off + c4 * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(u2f(ov[e]) * alpha);
            tmem_st32(tOt + lane_off + c4 * 32, ov);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(t));
      }
      // epilogue: O / l -> bf16, LSE
      if (ok && cnt > 0 && mbar_wait_warp(pv_done(t), (cnt - 1) & 1, kErrFwd, 0x420 + t)) {
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* orow = nullptr;
        if (row_ok) {
          if (a.seq) {
            const int p = i / a.n_loc;
            orow = static_cast<__nv_bfloat16*>(a.o.p[p]) +
                   (static_cast<int64_t>(i - p * a.n_loc) * (a.Hl * a.P) + r * a.Hl + h) * D;
          } else {
            orow = static_cast<__nv_bfloat16*>(a.o.p[r]) + (static_cast<int64_t>(i) * a.Hl + h) * D;
          }
        }
#pragma unroll 1
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t ov[32];
          tmem_ld32(tOt + lane_off + c4 * 32, ov);
          tmem_wait_ld();
          uint4 pk[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int e = 0; e < 16; ++e) pw[e] = pack_bf16x2(u2f(ov[2 * e]) * inv, u2f(ov[2 * e + 1]) * inv);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = pk[e];
          }
        }
        if (row_ok) a.lse.p[r][static_cast<int64_t>(h) * N + i] = (m_run + lg2_approx(l_run)) * kLn2;
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

// ---------------------------------------------------------------- host side
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

// 2D map over a [rows, row_elems] bf16 matrix with 128-byte-swizzled 64 x 128 boxes.
bool encode_rows(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t rows, int64_t row_elems) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_elems), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_elems * 2)};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const FwdArgs& a, int nranks, cudaStream_t stream) {
  using L = Layout<D>;
  cudaError_t e =
      cudaFuncSetAttribute(attn_fwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hl * nranks, a.num_m_blocks);
  attn_fwd_sm100_kernel<D><<<grid, kThreads, L::kAlloc, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fwd_sm100

namespace fwd_sm100 {
cudaError_t launch_common(const AttnShape& s, FwdArgs& a, cudaStream_t stream) {
  a.cu = s.cu_seqlens;
  a.num_seqs = s.num_seqs;
  a.N = s.N;
  a.Hl = s.Hl;
  a.Hkvl = s.Hkvl;
  a.group = s.Hl / s.Hkvl;
  a.scale_log2 = s.scale * kLog2e;
  a.rank_lo = s.rank_lo;
  a.num_m_blocks = (s.N + 2 * BM - 1) / (2 * BM);
  a.n_loc = s.N / s.P;
  a.P = s.P;
  const int nranks = s.rank_hi - s.rank_lo;
  return s.d == 64 ? launch_d<64>(a, nranks, stream) : launch_d<128>(a, nranks, stream);
}
}  // namespace fwd_sm100

cudaError_t launch_attn_fwd(const AttnShape& s, const void* const* q, const void* const* k, const void* const* v,
                            void* const* o, float* const* lse, cudaStream_t stream) {
  using namespace fwd_sm100;
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return cudaErrorNotSupported;
  FwdArgs a;   // ~6.5 KB, copied into the launch's parameter space
  memset(&a, 0, sizeof(a));
  for (int r = s.rank_lo; r < s.rank_hi; ++r) {
    if (!encode_rows(enc, &a.tq[r], q[r], s.N, static_cast<int64_t>(s.Hl) * s.d) ||
        !encode_rows(enc, &a.tk[r], k[r], s.N, static_cast<int64_t>(s.Hkvl) * s.d) ||
        !encode_rows(enc, &a.tv[r], v[r], s.N, static_cast<int64_t>(s.Hkvl) * s.d))
      return cudaErrorInvalidValue;
    a.o.p[r] = o[r];
    a.lse.p[r] = lse[r];
  }
  a.seq = 0;
  return launch_common(s, a, stream);
}

cudaError_t launch_attn_fwd_seq(const AttnShape& s, const void* const* q_seq, const void* const* k_seq,
                                const void* const* v_seq, void* const* o_seq, float* const* lse,
                                cudaStream_t stream) {
  using namespace fwd_sm100;
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return cudaErrorNotSupported;
  FwdArgs a;
  memset(&a, 0, sizeof(a));
  const int64_t n = s.N / s.P;
  const int64_t H = static_cast<int64_t>(s.Hl) * s.P, Hkv = static_cast<int64_t>(s.Hkvl) * s.P;
  for (int p = 0; p < s.P; ++p) {
    if (!encode_rows(enc, &a.tq[p], q_seq[p], n, H * s.d) || !encode_rows(enc, &a.tk[p], k_seq[p], n, Hkv * s.d) ||
        !encode_rows(enc, &a.tv[p], v_seq[p], n, Hkv * s.d))
      return cudaErrorInvalidValue;
    a.o.p[p] = o_seq[p];
  }
  for (int r = s.rank_lo; r < s.rank_hi; ++r) a.lse.p[r] = lse[r];
  a.seq = 1;
  return launch_common(s, a, stream);
}

}  // namespace uly
