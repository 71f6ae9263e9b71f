// One-pass attention backward for sm_100a (head dim 128): the dK/dV kernel
// also produces dQ, so S and dP are computed once per block pair (5 block GEMMs
// instead of the two-pass path's 7).
//
// One CTA per 128-key block of one key/value head: K and V stay in shared
// memory and 128-row blocks of Q and dO (with the rows' lse*log2(e) and D)
// stream through a 2-stage ring. Per streamed block, every GEMM is
// M = 128, N = 128 (the tensor pipe's full rate; N = 64 shared-memory-operand
// GEMMs run at about half of it):
//   S^T = K Q^T, dP^T = V dO^T          (SS MMAs into TMEM)
//   P^T, dS^T elementwise: one thread per key row and 64 query columns, the
//   two elementwise warpgroups on the two column halves of the same block;
//   P^T (bf16) goes back into TMEM over S^T, dS^T (bf16) into a 128-byte-
//   swizzled shared-memory tile
//   dV += P^T dO                          (TS MMA: A = P^T from TMEM)
//   dK += dS^T Q                          (SS MMA: A = dS^T from shared memory)
//   dQ^T_blk = K^T dS^T                   (SS MMA into the dP^T columns)
// TMEM (512 columns): dV, dK accumulators 128 each, S^T 128, dP^T 128. With
// S^T single-buffered, the next block's S^T is issued as soon as dV has read
// P^T, so it runs while the elementwise warps compute dS^T; dK reads dS^T
// from shared memory for that reason, not from the S^T columns.
// A dedicated dQ warpgroup reads dQ^T_blk back (TMEM lane = head-dim index,
// column = row), releases the columns for the next dP^T, and adds it from
// registers into an fp32 accumulator in global memory with 16-byte vector
// reductions (red.global.add.v4.f32): the L2 performs the sums, so no CTA
// waits on another. The order of those fp32 sums depends on timing, so dQ is
// not bit-reproducible from run to run (dK and dV are). A final kernel scales
// the accumulator by the softmax scale and writes bf16 dQ.
//
// Accumulator layout: per (rank, query head, 64-row block) one 32 KB block of
// 16 x 128 x 4 floats, element (row q, dim c) at ((q / 4) * 128 + c) * 4 + q % 4,
// the order in which one warp's 32 lanes (32 consecutive c) store 4 rows each
// as 16-byte vectors without bank conflicts.
//
// Shared memory: K, V 64 KB; ring 2 x 64 KB (+ 2 x 1 KB for lse*log2(e) and
// D of the stage's rows); dS^T 32 KB; barriers. That is about 226.1 KB of the
// 232,448 bytes a CTA may have, so the kernel relies on the dynamic shared
// memory base being within about 900 bytes of a 1024-byte boundary (it is at
// one on sm_100); the host checks this before choosing this kernel and the
// kernel reports kErrBwd site 0xA11 without touching anything if not.
// Included by attn_bwd_sm100.cu after the two-pass kernels (shares their
// constants, argument struct and helpers). The Q and dO tensor maps it is
// given have 128-row boxes.

namespace uly {
namespace bwd_sm100 {
namespace onepass {

constexpr int D = 128;
constexpr int QB = 128;       // streamed query rows per block
constexpr int NSTG = 2;
constexpr int kAccRows = 64;  // rows per fp32 dQ accumulator block
static_assert(QB == TB, "query blocks start on key-block boundaries");
// Four warpgroups: elementwise on query columns 0-63 / 64-127 of every block
// (warps 0-3, 4-7), the TMA producer (warp 8) and MMA issuer (warp 9) with two
// idle warps, and the dQ warpgroup (warps 12-15). 512 threads launch with 128
// registers each (all 65,536); the control warpgroup drops to kRegsOpCtl and
// the elementwise and dQ ones (the latter holds a 128-column row of dQ^T)
// rise to kRegsOpEw and kRegsOpDq: 2*128*144 + 128*72 + 128*152 = 65,536.
constexpr int kOpThreads = 512;
constexpr int kRegsOpEw = 144, kRegsOpCtl = 72, kRegsOpDq = 152;
static_assert(2 * 128 * kRegsOpEw + 128 * kRegsOpCtl + 128 * kRegsOpDq <= 65536, "register split above the launch");

struct Layout {
  static constexpr uint32_t kKV = TB * D * 2;          // 32 KB: K or V
  static constexpr uint32_t kBlk = QB * D * 2;         // 32 KB: one streamed Q or dO block
  static constexpr uint32_t kHalf = QB * 128;          // 16 KB: 64 head dims of a block
  static constexpr uint32_t kK = 0, kV = kKV;
  static constexpr uint32_t kRing = 2 * kKV;           // stage s: Q at +0, dO at +kBlk
  static constexpr uint32_t kDS = kRing + NSTG * 2 * kBlk;   // dS^T: query half j at +j * kDSh
  static constexpr uint32_t kDSh = TB * 64 * 2;        // 16 KB
  static constexpr uint32_t kVec = kDS + 2 * kDSh;     // stage s: lse2 at +0, D at +512
  static constexpr uint32_t kVecStage = 2 * QB * 4;
  static constexpr uint32_t kBars = kVec + NSTG * kVecStage;
  // kv_full, st_full[2], st_empty[2], s_full, s_free, p_full, dp_full, ds_full, dq_full, dq_free, acc_done
  static constexpr int kNumBars = 1 + 2 * NSTG + 8;
  static constexpr uint32_t kSlot = kBars + kNumBars * 8;
  static constexpr uint32_t kUsed = kSlot + 16;
  static constexpr uint32_t kAlloc = 232448;           // the per-CTA maximum on sm_100
};
static_assert(Layout::kUsed <= Layout::kAlloc, "one-pass backward does not fit in shared memory");

// *addr += {a, b, c, d} (fp32 bit patterns, 16-byte aligned), performed in the L2
ULY_DEV void red_add_v4(float* addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(__uint_as_float(a)),
               "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
               : "memory");
}
// An opaque copy of a descriptor: the per-MMA offsets are then added at issue
// time instead of being hoisted out of the block loop as dozens of live
// 64-bit registers (the MMA warp runs with few registers).
ULY_DEV uint64_t opaque(uint64_t d) {
  uint64_t r;
  asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(d));
  return r;
}
ULY_DEV void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __launch_bounds__(kOpThreads, 1) attn_bwd_onepass_kernel(const __grid_constant__ DkdvArgs a) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  if (sbase - raw + L::kUsed > L::kAlloc) {
    if (threadIdx.x == 0) report_error(kErrBwd, 0xA11);
    return;
  }
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + L::kBars;
  const uint32_t kv_full = bars;
  auto st_full = [&](int s) { return bars + 8u * (1 + s); };
  auto st_empty = [&](int s) { return bars + 8u * (1 + NSTG + s); };
  const uint32_t s_full = bars + 8u * (1 + 2 * NSTG);
  const uint32_t s_free = s_full + 8u;
  const uint32_t p_full = s_full + 16u;
  const uint32_t dp_full = s_full + 24u;
  const uint32_t ds_full = s_full + 32u;
  const uint32_t dq_full = s_full + 40u;
  const uint32_t dq_free = s_full + 48u;
  const uint32_t acc_done = s_full + 56u;
  volatile uint32_t* slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // kb_fast: blockIdx.x is the key block, so the CTAs resident together
  // belong to one (rank, kv head) and stream the same Q/dO blocks into the
  // same accumulator rows, which then stay in L2. Else blockIdx.x is the
  // (rank, kv head) and every pair's heaviest key blocks launch first (the
  // host picks; see launch_onepass).
  const int combo = a.kb_fast ? blockIdx.y : blockIdx.x;
  const int g = combo % a.Hkvl;
  const int r = a.rank_lo + combo / a.Hkvl;
  const int N = a.N;
  const int n0 = (a.kb_fast ? blockIdx.x : blockIdx.y) * TB;
  const int n_last = min(n0 + TB, N) - 1;
  const int doc_end_first = doc_end_of(a.cu, a.num_seqs, n0, N);
  const int m_end = doc_end_of(a.cu, a.num_seqs, n_last, N);
  const int rb_lo = n0 / QB;
  const int nrb = (m_end + QB - 1) / QB - rb_lo;
  const int T = a.group * nrb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bars + 8u * i, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(dq_free, 128);
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
  const uint32_t tDV = tmem, tDK = tmem + D, tS = tmem + 256u, tDP = tmem + 384u;

  if (warp >= 8 && warp < 12) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOpCtl));
  if (warp == kTmaWarp) {
    {
      auto shard_of = [&](int tok) { return a.seq ? tok / a.n_loc : r; };
      auto row_in = [&](int tok) { return a.seq ? tok - (tok / a.n_loc) * a.n_loc : tok; };
      // Q and dO: sequence shards (qdo_seq) or head shards (also in the
      // sequence-layout call, which may stage them there first)
      auto q_shard = [&](int tok) { return a.qdo_seq ? tok / a.n_loc : r; };
      auto q_row = [&](int tok) { return a.qdo_seq ? tok - (tok / a.n_loc) * a.n_loc : tok; };
      const int qx0 = a.qdo_seq ? r * a.Hl * D : 0, kx0 = a.seq ? (r * a.Hkvl + g) * D : g * D;
      if (!a.qdo_seq && lane == 0) {
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
        const int s = it % NSTG;
        if (!mbar_wait_warp(st_empty(s), ((it / NSTG) & 1) ^ 1, kErrBwd, 0xA00 + s)) break;
        const int h = g * a.group + it / nrb;
        const int m0 = (rb_lo + it % nrb) * QB;
        const uint32_t stg = sbase + L::kRing + s * 2 * L::kBlk;
        mbar_arrive_expect_tx_w(st_full(s), 2 * L::kBlk + L::kVecStage);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          tma_load_2d_w(stg + hf * L::kHalf, &a.tq[q_shard(m0)], st_full(s), qx0 + h * D + hf * 64, q_row(m0));
          tma_load_2d_w(stg + L::kBlk + hf * L::kHalf, &a.tdo[q_shard(m0)], st_full(s), qx0 + h * D + hf * 64,
                        q_row(m0));
        }
        const int64_t vo = (static_cast<int64_t>(r) * a.Hl + h) * a.Npad + m0;
        bulk_load_w(sbase + L::kVec + s * L::kVecStage, a.lse2 + vo, QB * 4, st_full(s));
        bulk_load_w(sbase + L::kVec + s * L::kVecStage + QB * 4, a.Dv + vo, QB * 4, st_full(s));
      }
      for (int k = it > NSTG ? it - NSTG : 0; k < it; ++k)
        mbar_wait_drain_w(st_full(k % NSTG), (k / NSTG) & 1, kErrBwd, 0xAF0);
      mbar_wait_drain_w(kv_full, 0, kErrBwd, 0xAF1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    {
      // Tensor-pipe order per block: dV(i) S(i+1) dK(i) dQ(i) dP(i+1). S(i+1)
      // overwrites the P^T that dV(i) reads, so it waits for dV(i) to finish;
      // dP(i+1) overwrites the dQ^T(i) columns, so it waits for the dQ
      // warpgroup to have read them.
      constexpr uint32_t idS = idesc_bf16_f32(TB, QB, 0, 0);   // S^T, dP^T: M=128 keys, N=128 rows
      constexpr uint32_t idV = idesc_bf16_f32(TB, D, 0, 1);    // dV (A = P^T in TMEM), dK (A = dS^T K-major)
      constexpr uint32_t idQ = idesc_bf16_f32(D, QB, 1, 1);    // dQ^T: M=128 dims, N=128 rows
      bool ok = mbar_wait_warp(kv_full, 0, kErrBwd, 0xA20);
      tc_fence_after();
      const uint64_t dK0 = smem_desc_sw128(sbase + L::kK, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sbase + L::kV, 16, 1024);
      const uint64_t dKmn = smem_desc_sw128(sbase + L::kK, TB * 128, 1024);   // K as the M-major A of dQ^T
      const uint64_t dRing0 = smem_desc_sw128(sbase + L::kRing, 16, 1024);
      const uint64_t dRingMN0 = smem_desc_sw128(sbase + L::kRing, L::kHalf, 1024);
      const uint64_t dDS0 = smem_desc_sw128(sbase + L::kDS, 16, 1024);          // dS^T, K-major A of dK
      const uint64_t dDSmn = smem_desc_sw128(sbase + L::kDS, L::kDSh, 1024);    // dS^T, N-major B of dQ^T
      // 16-wide K step kk of a 128-row operand stored as two 64-column halves
      auto kstep = [](int kk) { return static_cast<uint32_t>((kk / 4) * (128 * 128) + (kk % 4) * 32); };
      auto issue_s = [&](int it) {
        const uint64_t ad = opaque(dK0), qd = opaque(desc_adv(dRing0, (it % NSTG) * 2 * L::kBlk));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_w(tS, desc_adv(ad, kstep(kk)), desc_adv(qd, kstep(kk)), idS, kk > 0 ? 1u : 0u);
        mma_commit_w(s_full);
      };
      auto issue_dp = [&](int it) {
        const uint64_t ad = opaque(dV0), dod = opaque(desc_adv(dRing0, (it % NSTG) * 2 * L::kBlk + L::kBlk));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_w(tDP, desc_adv(ad, kstep(kk)), desc_adv(dod, kstep(kk)), idS, kk > 0 ? 1u : 0u);
        mma_commit_w(dp_full);
      };
      if (ok && T > 0) {
        if (!mbar_wait_warp(st_full(0), 0, kErrBwd, 0xA21)) ok = false;
        tc_fence_after();
        if (ok) {
          issue_s(0);
          issue_dp(0);
        }
      }
      for (int it = 0; it < T && ok; ++it) {
        const int ph = it & 1;
        const uint32_t stg_off = (it % NSTG) * 2 * L::kBlk;
        if (!mbar_wait_warp(p_full, ph, kErrBwd, 0xA30)) { ok = false; break; }
        tc_fence_after();
        {
          // dV += P^T dO: P^T of query half j sits in S^T columns 64j .. 64j+31
          const uint64_t dob = opaque(desc_adv(dRingMN0, stg_off + L::kBlk));
#pragma unroll
          for (int kk = 0; kk < QB / 16; ++kk)
            mma_ts_w(tDV, tS + (kk / 4) * 64 + (kk % 4) * 8, desc_adv(dob, kk * 2048), idV,
                     (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(s_free);
        }
        if (it + 1 < T) {
          const int nx = it + 1;
          if (!mbar_wait_warp(st_full(nx % NSTG), (nx / NSTG) & 1, kErrBwd, 0xA31)) { ok = false; break; }
          if (!mbar_wait_warp(s_free, ph, kErrBwd, 0xA32)) { ok = false; break; }
          tc_fence_after();
          issue_s(nx);
        }
        if (!mbar_wait_warp(ds_full, ph, kErrBwd, 0xA33)) { ok = false; break; }
        tc_fence_after();
        {
          const uint64_t qb = opaque(desc_adv(dRingMN0, stg_off)), ab = opaque(dDS0);
#pragma unroll
          for (int kk = 0; kk < QB / 16; ++kk)
            mma_ss_w(tDK, desc_adv(ab, kstep(kk)), desc_adv(qb, kk * 2048), idV, (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(st_empty(it % NSTG));     // Q(i) and dO(i) consumed
          const uint64_t kq = opaque(dKmn), dsq = opaque(dDSmn);
#pragma unroll
          for (int kk = 0; kk < TB / 16; ++kk)
            mma_ss_w(tDP, desc_adv(kq, kk * 2048), desc_adv(dsq, kk * 2048), idQ, kk > 0 ? 1u : 0u);
          mma_commit_w(dq_full);
        }
        if (it + 1 < T) {
          if (!mbar_wait_warp(dq_free, ph, kErrBwd, 0xA34)) { ok = false; break; }
          tc_fence_after();
          issue_dp(it + 1);
        }
      }
      mma_commit_w(acc_done);
      mbar_wait_drain_w(acc_done, 0, kErrBwd, 0xA50);
    }
    __syncwarp();
  }   // warps 10, 11: nothing to do
  } else if (warp >= 12) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsOpDq));
    // ------------------------------------------------------------ dQ
    // Block it's dQ^T (lane = head-dim index, column = row m0 + column) from
    // TMEM into registers, release the columns, add into the accumulator.
    const int lrow = 32 * (warp & 3) + lane;
    const uint32_t loff = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int64_t qblocks = a.Npad / kAccRows;
    for (int it = 0; it < T; ++it) {
      const int h = g * a.group + it / nrb;
      const int m0 = (rb_lo + it % nrb) * QB;
      if (!mbar_wait_warp(dq_full, it & 1, kErrBwd, 0xC30)) break;
      tc_fence_after();
      uint32_t dq[QB];
#pragma unroll
      for (int c = 0; c < QB / 32; ++c) tmem_ld32(tDP + loff + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&dq[32 * c]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(dq_free);
      float* dst =
          a.dqacc + ((static_cast<int64_t>(r) * a.Hl + h) * qblocks + m0 / kAccRows) * (kAccRows * D) + lrow * 4;
#pragma unroll
      for (int t = 0; t < QB / 4; ++t)
        red_add_v4(dst + (t / (kAccRows / 4)) * (kAccRows * D) + (t % (kAccRows / 4)) * (D * 4), dq[4 * t],
                   dq[4 * t + 1], dq[4 * t + 2], dq[4 * t + 3]);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsOpEw));
    // ------------------------------------------------------------ elementwise
    const int j = warp >> 2;                            // this warpgroup's query columns: 64j .. 64j+63
    const int lrow = 32 * (warp & 3) + lane;            // TMEM lane: key row, then head-dim index
    const uint32_t loff = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int key = n0 + lrow;
    const int kde = doc_end_of(a.cu, a.num_seqs, min(key, N - 1), N);
    const float sl2 = a.scale_log2;
    const uint32_t dsrow = sbase + L::kDS + j * L::kDSh + lrow * 128;
    const uint32_t swz = static_cast<uint32_t>(lrow & 7);
    const uint32_t tSj = tS + 64u * j + loff, tDPj = tDP + 64u * j + loff;
    bool ok = true;
    for (int it = 0; it < T; ++it) {
      const int s = it % NSTG;
      const int m0 = (rb_lo + it % nrb) * QB;
      const uint32_t vl = sbase + L::kVec + s * L::kVecStage + 256 * j, vd = vl + QB * 4;
      if (!mbar_wait_warp(st_full(s), (it / NSTG) & 1, kErrBwd, 0xB00)) { ok = false; break; }
      if (!mbar_wait_warp(s_full, it & 1, kErrBwd, 0xB10)) { ok = false; break; }
      tc_fence_after();
      uint32_t pv[64];
      tmem_ld32(tSj, *reinterpret_cast<uint32_t(*)[32]>(&pv[0]));
      tmem_ld32(tSj + 32, *reinterpret_cast<uint32_t(*)[32]>(&pv[32]));
      tmem_wait_ld();
      const bool need_mask = (m0 < n0 + TB - 1) || (m0 + QB > doc_end_first);
      const int lo = key - m0 - 64 * j;
      const uint32_t span = static_cast<uint32_t>(max(kde - key, 0));
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
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
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(u2f(pv[2 * c]), u2f(pv[2 * c + 1]));
        tmem_st32(tSj, pk);    // P^T over this warpgroup's own (already read) S^T columns
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      if (!mbar_wait_warp(dp_full, it & 1, kErrBwd, 0xB20)) { ok = false; break; }
      tc_fence_after();
      uint32_t ds[32];
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        uint32_t dp[32];
        tmem_ld32(tDPj + 32 * hc, dp);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 d4 = ld_shared_f4(vd + 4 * (32 * hc + c));
          const int cc = 32 * hc + c;
          const float d0 = u2f(pv[cc]) * (u2f(dp[c]) - d4.x);
          const float d1 = u2f(pv[cc + 1]) * (u2f(dp[c + 1]) - d4.y);
          const float d2 = u2f(pv[cc + 2]) * (u2f(dp[c + 2]) - d4.z);
          const float d3 = u2f(pv[cc + 3]) * (u2f(dp[c + 3]) - d4.w);
          ds[cc / 2] = pack_bf16x2(d0, d1);
          ds[cc / 2 + 1] = pack_bf16x2(d2, d3);
        }
      }
      tc_fence_before();
      // dS^T into the 128-byte-swizzled shared tile (A of dK, B of dQ^T): 8 chunks of 16 bytes
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(dsrow + ((static_cast<uint32_t>(c) ^ swz) << 4), ds[4 * c], ds[4 * c + 1], ds[4 * c + 2],
                     ds[4 * c + 3]);
      fence_proxy_async();
      mbar_arrive(ds_full);
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK
    if (ok && mbar_wait_warp(acc_done, 0, kErrBwd, 0xB50)) {
      tc_fence_after();
      const uint32_t src = (j == 0 ? tDV : tDK) + loff;
      const float mul = j == 0 ? 1.f : a.scale;
      const int kb = a.seq ? min(key, N - 1) / a.n_loc : r;
      const int64_t krow = a.seq ? (static_cast<int64_t>(key - kb * a.n_loc) * (a.Hkvl * a.P) + r * a.Hkvl + g)
                                 : (static_cast<int64_t>(key) * a.Hkvl + g);
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(j == 0 ? a.dv.p[kb] : a.dk.p[kb]) + krow * D;
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

// dQ = scale * accumulator, as bf16, into the head shards (seq == 0) or the
// sequence shards (seq == 1). One thread per (rank, head, 4 rows, 4 dims): it
// reads 4 float4 (64 contiguous bytes) and writes 4 rows x 8 bytes; a warp
// covers all 128 dims of 4 rows, so both sides are contiguous.
struct ConvArgs {
  const float* acc;
  RankPtrsMut dq;
  int N, Npad, Hl, rank_lo, nranks;
  float scale;
  int seq, n_loc, P;
};

__global__ void __launch_bounds__(256) dq_convert_kernel(const __grid_constant__ ConvArgs a) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int c4 = static_cast<int>(tid & 31);            // dims 4*c4 .. 4*c4+3
  const int64_t grp = tid >> 5;                          // (rank, head, 4-row group)
  const int64_t groups_per_head = a.Npad / 4;
  const int64_t total = groups_per_head * a.Hl * a.nranks;
  if (grp >= total) return;
  const int64_t rh = grp / groups_per_head;              // rank-in-range * Hl + head
  const int t = static_cast<int>(grp - rh * groups_per_head);   // 4-row group within the head
  const int rr = static_cast<int>(rh / a.Hl), h = static_cast<int>(rh - static_cast<int64_t>(rr) * a.Hl);
  const int r = a.rank_lo + rr;
  const int q0 = 4 * t;
  if (q0 >= a.N) return;
  // block (r, h, q0 / 64), position (q0 % 64) / 4 within it
  const float* src = a.acc + ((static_cast<int64_t>(r) * a.Hl + h) * (a.Npad / kAccRows) + q0 / kAccRows) *
                                 (kAccRows * D) +
                     ((q0 % kAccRows) / 4) * (D * 4) + c4 * 16;
  float4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __ldcs(reinterpret_cast<const float4*>(src) + i);   // dim 4*c4+i, rows q0..q0+3
  const float* vf = reinterpret_cast<const float*>(v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int q = q0 + k;
    if (q >= a.N) break;
    uint2 o;
    o.x = pack_bf16x2(vf[0 * 4 + k] * a.scale, vf[1 * 4 + k] * a.scale);
    o.y = pack_bf16x2(vf[2 * 4 + k] * a.scale, vf[3 * 4 + k] * a.scale);
    int buf = r;
    int64_t row = static_cast<int64_t>(q) * a.Hl + h;
    if (a.seq) {
      buf = q / a.n_loc;
      row = static_cast<int64_t>(q - buf * a.n_loc) * (a.Hl * a.P) + r * a.Hl + h;
    }
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.dq.p[buf]) + row * D + c4 * 4) = o;
  }
}

}  // namespace onepass
}  // namespace bwd_sm100
}  // namespace uly
