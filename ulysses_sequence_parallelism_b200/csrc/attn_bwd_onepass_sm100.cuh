// One-pass attention backward for sm_100a (head dim 128): the dK/dV kernel
// also produces dQ, so S and dP are computed once per block pair (5 block GEMMs
// instead of the two-pass path's 7).
//
// One CTA per 128-key block of one key/value head, as in the dK/dV kernel:
// K and V stay in shared memory and 64-row blocks of Q and dO stream through a
// 4-stage ring. Per streamed block:
//   S^T = K Q^T, dP^T = V dO^T               (SS MMAs, double-buffered in TMEM)
//   P^T, dS^T elementwise (one thread per key row); P^T and dS^T (bf16) into
//   TMEM over S^T, dS^T also into a 128-byte-swizzled shared-memory tile
//   dV += P^T dO                              (TS MMA)
//   dK += dS^T Q                              (TS MMA)
//   dQ^T_blk = K^T dS^T                       (SS MMA into the dP^T columns)
// A dedicated dQ warpgroup reads dQ^T_blk back (TMEM lane = head-dim index,
// column = row), releases the columns, and adds it straight from registers
// into an fp32 accumulator in global memory with 16-byte vector reductions
// (red.global.add.v4.f32): the L2 performs the sums, so no CTA waits on
// another, and the elementwise warpgroups go on to their next block without
// waiting for dQ (measured 1-2 % faster than having them do it). Nothing is staged in shared memory: shared-memory bandwidth, not
// the tensor pipe, bounds this kernel (every MMA here reads at least one
// operand from shared memory), so the dQ traffic stays out of it. The order of those fp32 sums
// depends on timing, so dQ is not bit-reproducible from run to run (dK and dV
// are). A final kernel scales the accumulator by the softmax scale and writes
// bf16 dQ.
//
// Accumulator layout: per (rank, query head, 64-row block) one 32 KB block of
// 16 x 128 x 4 floats, element (row q, dim c) at ((q / 4) * 128 + c) * 4 + q % 4,
// the order in which one warp's 32 lanes (32 consecutive c) store 4 rows each
// as 16-byte vectors without bank conflicts.
//
// Shared memory: K, V 64 KB; ring 4 x 32 KB (+ 4 x 512 B for lse*log2(e) and
// D of the stage's rows); dS^T 2 x 16 KB; barriers. That is about 231.6 KB of
// the 232,448 bytes a CTA may have, so the kernel relies on the dynamic shared
// memory base being within 800 bytes of a 1024-byte boundary (it is at one on
// sm_100); the kernel checks this first and reports kErrBwd site 0xA11
// without touching anything if not.
// Included by attn_bwd_sm100.cu after the two-pass kernels (shares their
// constants, argument struct and helpers).

namespace uly {
namespace bwd_sm100 {
namespace onepass {

constexpr int D = 128;
constexpr int NSTG = 4;
// Four warpgroups: elementwise for even / odd blocks (warps 0-3, 4-7), the
// TMA producer (warp 8) and MMA issuer (warp 9) with two idle warps, and the
// dQ warpgroup (warps 12-15), which takes each block's dQ^T out of TMEM and
// adds it into the fp32 accumulator in L2 so the elementwise warpgroups go
// straight on to their next block. 512 threads launch with 128 registers each
// (all 65,536); the control warpgroup drops to kRegsOpCtl and the dQ one to
// kRegsOpDq, and the elementwise ones rise to kRegsOpEw:
// 2*128*168 + 128*72 + 128*96 = 64,512 <= 65,536.
constexpr int kOpThreads = 512;
constexpr int kRegsOpEw = 168, kRegsOpCtl = 72, kRegsOpDq = 96;
static_assert(2 * 128 * kRegsOpEw + 128 * kRegsOpCtl + 128 * kRegsOpDq <= 65536, "register split above the launch");

struct Layout {
  static constexpr uint32_t kKV = TB * D * 2;          // 32 KB: K or V
  static constexpr uint32_t kBlk = SB * D * 2;         // 16 KB: one streamed Q or dO block
  static constexpr uint32_t kK = 0, kV = kKV;
  static constexpr uint32_t kRing = 2 * kKV;           // stage s: Q at +0, dO at +kBlk
  static constexpr uint32_t kDS = kRing + NSTG * 2 * kBlk;   // dS^T buffer b at +b * kDSb
  static constexpr uint32_t kDSb = TB * SB * 2;        // 16 KB
  static constexpr uint32_t kVec = kDS + 2 * kDSb;     // stage s: lse2 at +0, D at +256
  static constexpr uint32_t kBars = kVec + NSTG * 512;
  // kv_full, st_full[4], st_empty[4], s_full[2], dp_full[2], p_full[2], ds_full[2], dv_done[2],
  // dq_full[2], dq_free[2], acc_done
  static constexpr int kNumBars = 1 + 2 * NSTG + 14 + 1;
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
  auto s_full = [&](int b) { return bars + 8u * (1 + 2 * NSTG + b); };
  auto dp_full = [&](int b) { return bars + 8u * (3 + 2 * NSTG + b); };
  auto p_full = [&](int b) { return bars + 8u * (5 + 2 * NSTG + b); };
  auto ds_full = [&](int b) { return bars + 8u * (7 + 2 * NSTG + b); };
  auto dv_done = [&](int b) { return bars + 8u * (9 + 2 * NSTG + b); };
  auto dq_full = [&](int b) { return bars + 8u * (11 + 2 * NSTG + b); };
  auto dq_free = [&](int b) { return bars + 8u * (13 + 2 * NSTG + b); };
  const uint32_t acc_done = bars + 8u * (15 + 2 * NSTG);
  volatile uint32_t* slot = reinterpret_cast<volatile uint32_t*>(sgen + L::kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % a.Hkvl;
  const int r = a.rank_lo + blockIdx.x / a.Hkvl;
  const int N = a.N;
  const int n0 = blockIdx.y * TB;
  const int n_last = min(n0 + TB, N) - 1;
  const int doc_end_first = doc_end_of(a.cu, a.num_seqs, n0, N);
  const int m_end = doc_end_of(a.cu, a.num_seqs, n_last, N);
  const int rb_lo = n0 / SB;
  const int nrb = (m_end + SB - 1) / SB - rb_lo;
  const int T = a.group * nrb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bars + 8u * i, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(p_full(b), 128);
      mbar_init(ds_full(b), 128);
      mbar_init(dq_free(b), 128);
    }
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
  auto tDP = [&](int b) { return tmem + 256u + 128u * b + 64u; };   // dP^T, then dQ^T of the same block

  if (warp >= 8 && warp < 12) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOpCtl));
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
        const int s = it % NSTG;
        if (!mbar_wait_warp(st_empty(s), ((it / NSTG) & 1) ^ 1, kErrBwd, 0xA00 + s)) break;
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
      for (int k = it > NSTG ? it - NSTG : 0; k < it; ++k)
        mbar_wait_drain_w(st_full(k % NSTG), (k / NSTG) & 1, kErrBwd, 0xAF0);
      mbar_wait_drain_w(kv_full, 0, kErrBwd, 0xAF1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    {
      // Tensor-pipe order: dV(i) dP(i+1) dK(i) dQ(i) S(i+2) | dV(i+1) dP(i+2) ...
      // dP(i+1) reuses the columns of dQ(i-1), so it waits for that block's
      // drain; it is issued after dV(i) so the wait overlaps queued work.
      constexpr uint32_t idS = idesc_bf16_f32(TB, SB, 0, 0);   // S^T, dP^T: M=128 keys, N=64 rows
      constexpr uint32_t idA = idesc_bf16_f32(TB, D, 0, 1);    // dV, dK: M=128 keys, N=128 dims
      constexpr uint32_t idQ = idesc_bf16_f32(D, SB, 1, 1);    // dQ^T: M=128 dims, N=64 rows
      bool ok = mbar_wait_warp(kv_full, 0, kErrBwd, 0xA20);
      tc_fence_after();
      const uint64_t dK0 = smem_desc_sw128(sbase + L::kK, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sbase + L::kV, 16, 1024);
      const uint64_t dKmn = smem_desc_sw128(sbase + L::kK, TB * 128, 1024);   // K as the M-major A of dQ^T
      const uint64_t dRing0 = smem_desc_sw128(sbase + L::kRing, 16, 1024);
      const uint64_t dRingMN0 = smem_desc_sw128(sbase + L::kRing, SB * 128, 1024);
      const uint64_t dDSmn = smem_desc_sw128(sbase + L::kDS, 8192, 1024);       // dS^T, N-major B of dQ^T
      auto issue_s = [&](int it) {
        const uint64_t qd = desc_adv(dRing0, (it % NSTG) * 2 * L::kBlk);
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
        const uint64_t dod = desc_adv(dRing0, (it % NSTG) * 2 * L::kBlk + L::kBlk);
        const uint32_t dst = tDP(it & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk / 4) * (TB * 128) + (kk % 4) * 32;
          const uint32_t qo = (kk / 4) * (SB * 128) + (kk % 4) * 32;
          mma_ss_w(dst, desc_adv(dV0, ko), desc_adv(dod, qo), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(dp_full(it & 1));
      };
      if (ok && T > 0) {
        if (!mbar_wait_warp(st_full(0), 0, kErrBwd, 0xA21)) ok = false;
        tc_fence_after();
        if (ok) {
          issue_s(0);
          issue_dp(0);
        }
        if (ok && T > 1) {
          if (!mbar_wait_warp(st_full(1), 0, kErrBwd, 0xA21)) ok = false;
          tc_fence_after();
          if (ok) issue_s(1);
        }
      }
      for (int it = 0; it < T && ok; ++it) {
        const int b = it & 1;
        const uint32_t stg_off = (it % NSTG) * 2 * L::kBlk;
        if (!mbar_wait_warp(p_full(b), (it >> 1) & 1, kErrBwd, 0xA30)) { ok = false; break; }
        tc_fence_after();
        {
          const uint64_t dob = desc_adv(dRingMN0, stg_off + L::kBlk);
#pragma unroll
          for (int kk = 0; kk < SB / 16; ++kk)
            mma_ts_w(tDV, tS(b) + kk * 8, desc_adv(dob, kk * 2048), idA, (it > 0 || kk > 0) ? 1u : 0u);
        }
        if (it + 1 < T) {
          const int nx = it + 1;
          if (!mbar_wait_warp(st_full(nx % NSTG), (nx / NSTG) & 1, kErrBwd, 0xA31)) { ok = false; break; }
          if (it >= 1 && !mbar_wait_warp(dq_free(b ^ 1), ((it - 1) >> 1) & 1, kErrBwd, 0xA32)) { ok = false; break; }
          tc_fence_after();
          issue_dp(nx);
        }
        if (!mbar_wait_warp(ds_full(b), (it >> 1) & 1, kErrBwd, 0xA33)) { ok = false; break; }
        tc_fence_after();
        {
          const uint64_t qb = desc_adv(dRingMN0, stg_off);
#pragma unroll
          for (int kk = 0; kk < SB / 16; ++kk)
            mma_ts_w(tDK, tS(b) + 32 + kk * 8, desc_adv(qb, kk * 2048), idA, (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(dv_done(b));     // P^T and dS^T (both in the S^T columns) consumed
          const uint64_t dsB = desc_adv(dDSmn, b * L::kDSb);
#pragma unroll
          for (int kk = 0; kk < TB / 16; ++kk)
            mma_ss_w(tDP(b), desc_adv(dKmn, kk * 2048), desc_adv(dsB, kk * 2048), idQ, kk > 0 ? 1u : 0u);
          mma_commit_w(dq_full(b));
          mma_commit_w(st_empty(it % NSTG));     // dQ^T(i) was the stage's last reader
        }
        if (it + 2 < T) {
          const int nx = it + 2;
          if (!mbar_wait_warp(st_full(nx % NSTG), (nx / NSTG) & 1, kErrBwd, 0xA34)) { ok = false; break; }
          if (!mbar_wait_warp(dv_done(b), (it >> 1) & 1, kErrBwd, 0xA35)) { ok = false; break; }
          tc_fence_after();
          issue_s(nx);
        }
      }
      mma_commit_w(acc_done);
      mbar_wait_drain_w(acc_done, 0, kErrBwd, 0xA50);
    }
    __syncwarp();
  }   // warps 10, 11: nothing to do
  } else if (warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOpDq));
    // ------------------------------------------------------------ dQ
    // Block it's dQ^T (lane = head-dim index, column = row m0 + column) from
    // TMEM into registers, release the columns, add into the accumulator.
    const int lrow = 32 * (warp & 3) + lane;
    const uint32_t loff = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int64_t qblocks = a.Npad / SB;
    for (int it = 0; it < T; ++it) {
      const int b = it & 1;
      const int h = g * a.group + it / nrb;
      const int m0 = (rb_lo + it % nrb) * SB;
      if (!mbar_wait_warp(dq_full(b), (it >> 1) & 1, kErrBwd, 0xC30)) break;
      tc_fence_after();
      uint32_t dq[SB];
      tmem_ld32(tDP(b) + loff, *reinterpret_cast<uint32_t(*)[32]>(&dq[0]));
      tmem_ld32(tDP(b) + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&dq[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(dq_free(b));
      float* dst = a.dqacc + ((static_cast<int64_t>(r) * a.Hl + h) * qblocks + m0 / SB) * (SB * D) + lrow * 4;
#pragma unroll
      for (int t = 0; t < SB / 4; ++t)
        red_add_v4(dst + t * (D * 4), dq[4 * t], dq[4 * t + 1], dq[4 * t + 2], dq[4 * t + 3]);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsOpEw));
    // ------------------------------------------------------------ elementwise
    const int b = warp >> 2;                            // this warpgroup's blocks: it % 2 == b
    const int lrow = 32 * (warp & 3) + lane;            // TMEM lane: key row, then head-dim index
    const uint32_t loff = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int key = n0 + lrow;
    const int kde = doc_end_of(a.cu, a.num_seqs, min(key, N - 1), N);
    const float sl2 = a.scale_log2;
    const uint32_t dsrow = sbase + L::kDS + b * L::kDSb + lrow * 128;
    const uint32_t swz = static_cast<uint32_t>(lrow & 7);
    const int64_t qblocks = a.Npad / SB;
    bool ok = true;
    for (int it = b; it < T; it += 2) {
      const int s = it % NSTG;
      const int h = g * a.group + it / nrb;
      const int m0 = (rb_lo + it % nrb) * SB;
      const uint32_t vl = sbase + L::kVec + s * 512, vd = vl + 256;
      if (!mbar_wait_warp(st_full(s), (it / NSTG) & 1, kErrBwd, 0xB00)) { ok = false; break; }
      if (!mbar_wait_warp(s_full(b), (it >> 1) & 1, kErrBwd, 0xB10)) { ok = false; break; }
      tc_fence_after();
      uint32_t pv[SB];
      tmem_ld32(tS(b) + loff, *reinterpret_cast<uint32_t(*)[32]>(&pv[0]));
      tmem_ld32(tS(b) + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&pv[32]));
      tmem_wait_ld();
      const bool need_mask = (m0 < n0 + TB - 1) || (m0 + SB > doc_end_first);
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
      {
        uint32_t pk[SB / 2];
#pragma unroll
        for (int c = 0; c < SB / 2; ++c) pk[c] = pack_bf16x2(u2f(pv[2 * c]), u2f(pv[2 * c + 1]));
        tmem_st32(tS(b) + loff, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(b));
      if (!mbar_wait_warp(dp_full(b), (it >> 1) & 1, kErrBwd, 0xB20)) { ok = false; break; }
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
        dp[c / 2] = pack_bf16x2(d0, d1);
        dp[c / 2 + 1] = pack_bf16x2(d2, d3);
      }
      // dS^T as bf16 into the upper half of the S^T columns (A of the dK MMA) ...
      tmem_st32(tS(b) + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_wait_st();
      // ... and into the 128-byte-swizzled shared tile (B of the dQ^T MMA): 8 chunks of 16 bytes
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(dsrow + ((static_cast<uint32_t>(j) ^ swz) << 4), dp[4 * j], dp[4 * j + 1], dp[4 * j + 2],
                     dp[4 * j + 3]);
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(ds_full(b));
      // dQ^T of this block is the dQ warpgroup's
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK
    if (ok && mbar_wait_warp(acc_done, 0, kErrBwd, 0xB50)) {
      tc_fence_after();
      const uint32_t src = (b == 0 ? tDV : tDK) + loff;
      const float mul = b == 0 ? 1.f : a.scale;
      const int kb = a.seq ? min(key, N - 1) / a.n_loc : r;
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
  const float* src = a.acc + ((static_cast<int64_t>(r) * a.Hl + h) * (a.Npad / SB) + q0 / SB) * (SB * D) +
                     ((q0 % SB) / 4) * (D * 4) + c4 * 16;
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
