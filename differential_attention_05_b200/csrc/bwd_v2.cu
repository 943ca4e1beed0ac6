// bwd_v2.cu -- backward of the V2 prefill (bf16, d = 128) on the sm_100a tensor cores.
//
// The gradient is the forward's calculus (backward.cu states it). Notation per pair u
// (query heads 2u, 2u+1 over KV head g), scores S_b = Q_b K^T (raw), P_b = 2^(S_b sl2 -
// lse_b) with sl2 = log2(e)/sqrt(d) and lse_b the row's log2-domain log-sum-exp:
//   dP = dO V^T (the same for both branches),  dS_1 = P_1 o (dP - delta_1),
//   dS_2 = -lambda P_2 o (dP - delta_2),       delta_b = rowsum(dO o (P_b V)),
//   dV  = sum_u (P_1 - lambda P_2)^T dO,       dK = sum_u (dS_1^T Q_1 + dS_2^T Q_2) / sqrt(d),
//   dQ_b = dS_b K / sqrt(d).
// Three launches besides the fixed-order dlambda sum:
//   1. the forward kernel in its statistics mode (prefill_v2.cu) writes lse_1, lse_2,
//      delta_1, delta_2 and the dlambda share of every (query, pair);
//   2. bwd_v2_dkdv_kernel: one CTA per (128-key tile, KV head, batch entry) walks the pairs
//      of the GQA group and the 64-query tiles that see its keys. Per step the tensor core
//      computes S^T = K [Q_1; Q_2]^T (both branches stacked, N = 128) and dP^T = V dO^T;
//      the row threads (thread = key = TMEM lane) write (P_1 - lambda P_2)^T in bf16 to a
//      shared tile and [dS_1^T | dS_2^T] in bf16 to TMEM, and the tensor core accumulates
//      dV += (P_1 - lambda P_2)^T dO and dK += [dS_1^T | dS_2^T] [Q_1; Q_2] in TMEM (B = the
//      same shared tiles read MN-major). The next step's S^T and dP^T are issued as soon as
//      the rows have read this step's, so they run while the rows work;
//   3. bwd_v2_dq_kernel: one CTA per (64-query tile, pair, batch entry) walks the 128-key
//      tiles its queries see: S = [Q_1; Q_2] K^T and dP = [dO; dO] V^T (branches stacked in
//      the M = 128 rows), dS_b in bf16 into TMEM, dQ += dS K.
// V1 (d = 64, branches with their own keys K_1, K_2 and one value of width 2d) runs the same
// kernels: its key row is (K_1 | K_2), 128 wide, and the query tile is laid out zero-padded,
// rows 0-63 = (Q_1 | 0), rows 64-127 = (0 | Q_2), so one K = 128 MMA chain gives both
// branches' scores, dK = [dS_1^T | dS_2^T] [Q_1 0; 0 Q_2] is (dK_1 | dK_2) in the key layout,
// and dQ_b is the branch's own half of dS [K_1 | K_2]. Its statistics pass (the V1 forward
// kernel, prefill_v1.cu) also takes dy back through the per-head norm and writes that dO in
// bf16, which the kernels read in place of dy.
// No atomics: every dK/dV row and every dQ row is summed inside one CTA in a fixed order.
// The dQ kernel runs on a second stream beside the dK/dV kernel (see SideStream).
// Warps 0-15 (four warpgroups, each taking a quarter of a step's columns) form the per-row
// arithmetic, warp 16 issues the TMA loads (128-byte swizzle, no multicast) and the 1-D bulk
// copy of the statistics, warp 17 owns TMEM and every MMA.
// Every mbarrier wait is bounded as in the forward kernels.
#include "common.cuh"
#include "kernels.h"
#include "tma_host.cuh"

#include <mutex>
#include <type_traits>

namespace diffattn {

namespace {
constexpr int BLK = 128 * 128;   // [128 rows x 64 bf16] 128-byte-swizzled block (16 KB)
constexpr int HBLK = 64 * 128;   // [64 rows x 64 bf16] (8 KB)
constexpr unsigned FULL = 0xffffffffu;
// warps 0 .. 4 RW - 1: RW warpgroups of per-row arithmetic, each taking a quarter of a step's
// columns (so four warps share every TMEM lane quarter and hide each other's latency); then
// the TMA warp and the MMA warp
constexpr int RW = 4;
constexpr int NUM_THREADS = 128 * RW + 64;
constexpr int W_TMA = 4 * RW, W_MMA = 4 * RW + 1;
constexpr int TMEM_COLS = 512;

struct BwdMaps {
  CUtensorMap q, k, v, dy;
};

__device__ __forceinline__ uint64_t desc_at(uint64_t desc, uint32_t bytes) {
  return desc + (uint64_t)(bytes >> 4);
}

// does query i (at position i + Nk - N) attend key j
__device__ __forceinline__ bool visible(const PrefillArgs& a, int i, int j) {
  if (i >= a.N || j >= a.Nk) return false;
  if (!a.causal) return true;
  const int pos = i + a.Nk - a.N;
  return j <= pos && (a.window <= 0 || j > pos - a.window);
}

// is every (query, key) pair of queries q0 .. q0+nq-1 and keys k0 .. k0+nk-1 visible
__device__ __forceinline__ bool tile_visible(const PrefillArgs& a, int q0, int nq, int k0, int nk) {
  if (q0 + nq > a.N || k0 + nk > a.Nk) return false;
  if (!a.causal) return true;
  const int pos_lo = q0 + a.Nk - a.N, pos_hi = pos_lo + nq - 1;
  return k0 + nk - 1 <= pos_lo && (a.window <= 0 || k0 > pos_hi - a.window);
}

// ----------------------------------------------------------------------------- dK, dV
namespace kv {
constexpr int KT = 128, QT = 64;
// Two rings: [Q_1; Q_2] of a step (read by its first MMA, S^T, and its last, dK) three deep,
// so that the next step's copy never waits for the step before it to finish; dO and the
// statistics rows (read by dP^T, the row threads and dV) two deep.
constexpr int Q_STAGES = 3, D_STAGES = 2;
constexpr int K_OFF = 0, V_OFF = 2 * BLK;
constexpr int Q_OFF = 4 * BLK;                       // Q_STAGES x [Q_1; Q_2] (32 KB)
constexpr int D_OFF = Q_OFF + Q_STAGES * 2 * BLK;    // D_STAGES x (dO 16 KB + statistics 1 KB)
constexpr int STS = 2 * HBLK;                        // the statistics inside a dO stage
constexpr int D_STAGE = 2 * HBLK + 1024;
// (P_1 - lambda P_2)^T of a step in bf16, [128 keys x 64 queries] 128-byte swizzled: the A
// operand of the dV MMA, written by the row threads
constexpr int PC_OFF = D_OFF + D_STAGES * D_STAGE;
constexpr int MISC_OFF = PC_OFF + BLK;
constexpr int SMEM_BYTES = MISC_OFF + 1024 + 1024;
// TMEM columns: S^T (both branches), dP^T, [dS_1^T | dS_2^T] in bf16, dV, dK
constexpr int C_S = 0, C_DP = 128, C_DS = 192, C_DV = 256, C_DK = 384;
struct Misc {
  uint64_t kv_full, q_full[Q_STAGES], q_empty[Q_STAGES], d_full[D_STAGES], d_empty[D_STAGES];
  uint64_t s_full, p_full, o_full;
  uint64_t s_read;    // every row thread has read the step's S^T and dP^T columns
  uint64_t acc_done;  // the dV and dK MMAs of a step have completed (they read P and dS)
  uint32_t tmem_base;
  int abort;
};
static_assert(D_STAGE % 1024 == 0 && PC_OFF % 1024 == 0 && sizeof(Misc) <= 1024, "layout");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
}  // namespace kv
}  // namespace

template <bool V1>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_v2_dkdv_kernel(const __grid_constant__ BwdMaps maps, const BwdArgs g) {
  using namespace kv;
  const PrefillArgs& a = g.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + MISC_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_kt = a.Hkv * a.B;
  const int kt = (int)(blockIdx.x / per_kt);  // causal: key tile 0 sees the most queries
  const int gk = (int)(blockIdx.x % per_kt) % a.Hkv;
  const int b = (int)(blockIdx.x % per_kt) / a.Hkv;
  const int k0 = kt * KT;
  const int off = a.Nk - a.N;
  // queries that see a key of this tile, in 64-query tiles, for every pair of the group
  int i_lo = 0, i_hi = a.N - 1;
  if (a.causal) {
    i_lo = max(0, k0 - off);
    if (a.window > 0) i_hi = min(a.N - 1, k0 + KT - 1 - off + a.window - 1);
  }
  const int qt_lo = i_lo / QT;
  const int n_qt = i_hi >= i_lo ? i_hi / QT - qt_lo + 1 : 0;
  const int pairs = V1 ? 1 : a.group / 2, u0 = gk * pairs;
  const int n_steps = n_qt * pairs;  // step t: pair u0 + t / n_qt, query tile qt_lo + t % n_qt

  if (threadIdx.x == 0) {
    mbar_init(&ms.kv_full, 1);
    for (int s = 0; s < Q_STAGES; ++s) {
      mbar_init(&ms.q_full[s], 1);
      mbar_init(&ms.q_empty[s], 1);
    }
    for (int s = 0; s < D_STAGES; ++s) {
      mbar_init(&ms.d_full[s], 1);
      mbar_init(&ms.d_empty[s], 1);
    }
    mbar_init(&ms.s_full, 1);
    mbar_init(&ms.p_full, 4 * RW);  // one arrival per row warp
    mbar_init(&ms.o_full, 1);
    mbar_init(&ms.s_read, 4 * RW);
    mbar_init(&ms.acc_done, 1);
    ms.abort = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(&ms.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (V1) {
    // the zero quadrants of every stage's query tile (block 0 rows 64-127, block 1 rows
    // 0-63); the copies never write them
    for (int i = threadIdx.x; i < Q_STAGES * 2 * (HBLK / 16); i += NUM_THREADS) {
      const int st = i / (2 * (HBLK / 16)), r = i % (2 * (HBLK / 16));
      const int o = r < HBLK / 16 ? HBLK + 16 * r : BLK + 16 * (r - HBLK / 16);
      *reinterpret_cast<uint4*>(smem + Q_OFF + st * 2 * BLK + o) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  volatile int* abort_flag = &ms.abort;
  const int rows = a.N + 64;  // statistics rows per (batch entry, unit)

  if (warp == W_TMA) {
    if (lane == 0) {
      // ------------------------------ TMA producer -----------------------------------
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      tma_prefetch_desc(&maps.dy);
      mbar_arrive_expect_tx(&ms.kv_full, 4 * BLK);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_4d(smem + K_OFF + hf * BLK, &maps.k, &ms.kv_full, 64 * hf, gk, k0, b);
        tma_load_4d(smem + V_OFF + hf * BLK, &maps.v, &ms.kv_full, 64 * hf, gk, k0, b);
      }
      int q_issued = 0, d_issued = 0;
      for (int t = 0; t < n_steps && !*abort_flag; ++t) {
        const int u = u0 + t / n_qt, q0 = (qt_lo + t % n_qt) * QT;
        const int sq = t % Q_STAGES, sd = t % D_STAGES;
        if (!mbar_wait(&ms.q_empty[sq], ((t / Q_STAGES) & 1) ^ 1, abort_flag)) break;
        uint8_t* qs = smem + Q_OFF + sq * 2 * BLK;
        mbar_arrive_expect_tx(&ms.q_full[sq], V1 ? 2 * HBLK : 2 * BLK);
        for (int hf = 0; hf < 2; ++hf) {
          if (V1) {
            // (Q_1 | 0) in rows 0-63, (0 | Q_2) in rows 64-127: block hf gets branch hf
            tma_load_4d(qs + hf * BLK + hf * HBLK, &maps.q, &ms.q_full[sq], 64 * hf, u, q0, b);
          } else {
            // [Q_1; Q_2]: rows 0-63 branch 1, rows 64-127 branch 2 of each 64-column block
            tma_load_4d(qs + hf * BLK, &maps.q, &ms.q_full[sq], 64 * hf, 2 * u, q0, b);
            tma_load_4d(qs + hf * BLK + 64 * 128, &maps.q, &ms.q_full[sq], 64 * hf, 2 * u + 1, q0, b);
          }
        }
        q_issued = t + 1;
        if (!mbar_wait(&ms.d_empty[sd], ((t / D_STAGES) & 1) ^ 1, abort_flag)) break;
        uint8_t* ds = smem + D_OFF + sd * D_STAGE;
        // (w_st starts the workspace, so its offsets are workspace offsets)
        const int64_t st_off = (((int64_t)b * a.units + u) * rows + q0) * 4;
        const bool st_ok = in_bounds((g.w_st - g.w_base) + st_off, 256, g.ext_ws, a.dev_status, a.dbg_status);
        mbar_arrive_expect_tx(&ms.d_full[sd], 2 * HBLK + (st_ok ? 1024 : 0));
        for (int hf = 0; hf < 2; ++hf)
          tma_load_4d(ds + hf * HBLK, &maps.dy, &ms.d_full[sd], 64 * hf, u, q0, b);
        if (st_ok) bulk_load(ds + STS, g.w_st + st_off, 1024, &ms.d_full[sd]);
        d_issued = t + 1;
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA's shared memory goes away
        mbar_wait_drain(&ms.kv_full, 0);
        for (int t = max(0, q_issued - Q_STAGES); t < q_issued; ++t)
          mbar_wait_drain(&ms.q_full[t % Q_STAGES], (t / Q_STAGES) & 1);
        for (int t = max(0, d_issued - D_STAGES); t < d_issued; ++t)
          mbar_wait_drain(&ms.d_full[t % D_STAGES], (t / D_STAGES) & 1);
      }
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      // ------------------------------ MMA issuer -------------------------------------
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_DP = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, 128, false, true);
      const uint64_t kdesc = sw128_desc(smem_u32(smem + K_OFF), 16, 1024);
      const uint64_t vdesc = sw128_desc(smem_u32(smem + V_OFF), 16, 1024);
      // S^T of step t (both branches stacked, N = 128) into columns 0..127
      auto issue_st = [&](int t) {
        const uint64_t qd = sw128_desc(smem_u32(smem + Q_OFF + (t % Q_STAGES) * 2 * BLK), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk >> 2) * BLK + (kk & 3) * 32;
          umma_ss(tmem + C_S, desc_at(kdesc, o), desc_at(qd, o), IDESC_S, kk > 0);
        }
      };
      const uint64_t pcdesc = sw128_desc(smem_u32(smem + PC_OFF), 16, 1024);
      // dP^T of step t (N = 64) into columns 128..191, then the step is complete
      auto issue_dp = [&](int t) {
        const uint64_t dd = sw128_desc(smem_u32(smem + D_OFF + (t % D_STAGES) * D_STAGE), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk >> 2) * BLK + (kk & 3) * 32;
          const uint32_t od = (kk >> 2) * HBLK + (kk & 3) * 32;
          umma_ss(tmem + C_DP, desc_at(vdesc, o), desc_at(dd, od), IDESC_DP, kk > 0);
        }
        tc_commit(&ms.s_full);
      };
      auto issue_dv_dk = [&](int t) {
        // the same tiles read MN-major: K index = query (16 rows = 2048 B per step)
        const uint64_t dmn = sw128_desc(smem_u32(smem + D_OFF + (t % D_STAGES) * D_STAGE), HBLK, 1024);
        const uint64_t qmn = sw128_desc(smem_u32(smem + Q_OFF + (t % Q_STAGES) * 2 * BLK), BLK, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tmem + C_DV, desc_at(pcdesc, kk * 32), desc_at(dmn, kk * 2048), IDESC_ACC,
                  (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&ms.d_empty[t % D_STAGES]);  // dO and the statistics of step t are done with
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + C_DK, tmem + C_DS + kk * 8, desc_at(qmn, kk * 2048), IDESC_ACC,
                  (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&ms.q_empty[t % Q_STAGES]);
        tc_commit(&ms.acc_done);
      };
      // Per step t: S^T(t+1) and dP^T(t+1) as soon as the row threads have read step t's
      // columns, so that they run while the rows work on step t; then dV, dK of step t once
      // their operands are written. (The issuing thread is held at the tensor core's pace,
      // so this order is also the order the tensor core runs them in.)
      bool ok = mbar_wait(&ms.kv_full, 0, abort_flag);
      if (ok && n_steps > 0) {
        ok = mbar_wait(&ms.q_full[0], 0, abort_flag) && mbar_wait(&ms.d_full[0], 0, abort_flag);
        if (ok) {
          tc_fence_after();
          issue_st(0);
          issue_dp(0);
        }
      }
      for (int t = 0; t < n_steps && ok; ++t) {
        if (t + 1 < n_steps) {
          if (!(ok = mbar_wait(&ms.s_read, t & 1, abort_flag))) break;
          const int n = t + 1;
          if (!(ok = mbar_wait(&ms.q_full[n % Q_STAGES], (n / Q_STAGES) & 1, abort_flag))) break;
          tc_fence_after();
          issue_st(n);
          if (!(ok = mbar_wait(&ms.d_full[n % D_STAGES], (n / D_STAGES) & 1, abort_flag))) break;
          tc_fence_after();
          issue_dp(n);
        }
        if (!(ok = mbar_wait(&ms.p_full, t & 1, abort_flag))) break;
        tc_fence_after();
        issue_dv_dk(t);
      }
      // arrives once every MMA issued above has completed (also on an abort)
      tc_commit(&ms.o_full);
    }
  } else {
    // ------------------------- per-key arithmetic (warps 0 .. 4 RW - 1) --------------
    // warpgroup wgr takes queries 16 wgr .. 16 wgr + 15 of every 64-query step
    static_assert(RW == 4, "one 16-query chunk per row warpgroup");
    const int wgr = warp >> 2;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int kr = (warp & 3) * 32 + lane;  // this thread's key row (TMEM lane)
    const int j = k0 + kr;
    // this warpgroup's 16 queries of the key row in the swizzled P tile: 16-byte chunks
    // 2 wgr and 2 wgr + 1 of the row's 128 bytes
    uint8_t* pc_row = smem + PC_OFF + kr * 128;
    const int pc_c0 = ((2 * wgr) ^ (kr & 7)) << 4, pc_c1 = ((2 * wgr + 1) ^ (kr & 7)) << 4;
    const float sl2 = 1.4426950408889634f * rsqrtf((float)a.d);
    bool ok = true;
    for (int t = 0; t < n_steps; ++t) {
      const int sd = t % D_STAGES;
      const int u = u0 + t / n_qt, q0 = (qt_lo + t % n_qt) * QT;
      const float lam = a.lambda[u];
      if (ok) ok = mbar_wait(&ms.d_full[sd], (t / D_STAGES) & 1, abort_flag);
      if (ok) ok = mbar_wait(&ms.s_full, t & 1, abort_flag);
      if (!(ok = __all_sync(FULL, ok))) break;
      tc_fence_after();
      const float4* sts = reinterpret_cast<const float4*>(smem + D_OFF + sd * D_STAGE + STS);
      // inside the visible region (most steps of a causal problem) no pair needs a mask
      const bool full = tile_visible(a, q0, QT, k0, KT);
      auto chunk = [&](auto all_visible) {
        const int c = wgr;
        float s1[16], s2[16], dp[16];
        tmem_ld16f(lane_addr + kv::C_S + 16 * c, s1);
        tmem_ld16f(lane_addr + kv::C_S + 64 + 16 * c, s2);
        tmem_ld16f(lane_addr + kv::C_DP + 16 * c, dp);
        tmem_wait_ld();
        // the next step's S^T and dP^T may now overwrite their columns (one arrival per warp:
        // 512 single-thread arrivals on one barrier serialise)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms.s_read);
        uint32_t pc[8], d1[8], d2[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float vpc[2], vd1[2], vd2[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int qq = 16 * c + e + x;
            const float4 st = sts[qq];
            const bool vis = decltype(all_visible)::value || visible(a, q0 + qq, j);
            const float p1 = vis ? ex2(s1[e + x] * sl2 - st.x) : 0.f;
            const float p2 = vis ? ex2(s2[e + x] * sl2 - st.y) : 0.f;
            vpc[x] = p1 - lam * p2;
            vd1[x] = vis ? p1 * (dp[e + x] - st.z) : 0.f;
            vd2[x] = vis ? -lam * p2 * (dp[e + x] - st.w) : 0.f;
          }
          pc[e / 2] = pack_bf16(vpc[0], vpc[1]);
          d1[e / 2] = pack_bf16(vd1[0], vd1[1]);
          d2[e / 2] = pack_bf16(vd2[0], vd2[1]);
        }
        // P and dS of step t replace those of step t - 1 once its dV, dK MMAs are done
        if (t > 0) {
          if (ok) ok = mbar_wait(&ms.acc_done, (t - 1) & 1, abort_flag);
          if (!(ok = __all_sync(FULL, ok))) return;
          tc_fence_after();
        }
        // P_1 - lambda P_2 into the shared tile; dS_1, dS_2 into their 8-column slots of the
        // dS block
        *reinterpret_cast<uint4*>(pc_row + pc_c0) = make_uint4(pc[0], pc[1], pc[2], pc[3]);
        *reinterpret_cast<uint4*>(pc_row + pc_c1) = make_uint4(pc[4], pc[5], pc[6], pc[7]);
        tmem_st8(lane_addr + kv::C_DS + 8 * c, d1);
        tmem_st8(lane_addr + kv::C_DS + 32 + 8 * c, d2);
      };
      if (full) chunk(std::true_type{});
      else chunk(std::false_type{});
      if (!ok) break;
      tmem_wait_st();
      // the shared stores above become visible to the tensor core's operand reads
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.p_full);
    }
    // ------------------------------- epilogue ----------------------------------------
    if (ok) ok = mbar_wait(&ms.o_full, 0, abort_flag);
    ok = __all_sync(FULL, ok);
    // the TMEM loads run on the whole warp (they are warp-collective); only the stores
    // depend on the key being inside the sequence
    if (ok) {
      const float scale = rsqrtf((float)a.d);
      const int64_t row = ((int64_t)b * a.Nk + (j < a.Nk ? j : 0)) * a.Hkv + gk;
      const bool store = j < a.Nk && in_bounds(row * 128, 128, g.ext_dv, a.dev_status, a.dbg_status) &&
                         in_bounds(row * 128, 128, g.ext_dk, a.dev_status, a.dbg_status);
      float4* dv4 = reinterpret_cast<float4*>(g.dv + row * 128);
      float4* dk4 = reinterpret_cast<float4*>(g.dk + row * 128);
      const int c = wgr;  // this warpgroup's 32 columns of dV and dK
      if (n_steps > 0) {
        tc_fence_after();
        float x[32], y[32];
        tmem_ld32f(lane_addr + C_DV + 32 * c, x);
        tmem_ld32f(lane_addr + C_DK + 32 * c, y);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            dv4[(32 * c + e) / 4] = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
            dk4[(32 * c + e) / 4] = make_float4(y[e] * scale, y[e + 1] * scale,
                                                y[e + 2] * scale, y[e + 3] * scale);
          }
        }
      } else if (store) {
        for (int e = 0; e < 8; ++e) dv4[8 * c + e] = dk4[8 * c + e] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    if (*abort_flag) {
      mbar_wait_drain(&ms.o_full, 0);
      if (lane == 0) report_status(a.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ----------------------------------------------------------------------------- dQ
namespace {
namespace dqk {
constexpr int QT = 64, KT = 128;
// Two rings: a step's K tile (read by its first MMA, S, and its last, dQ) three deep, so
// that the next step's copy never waits for the step before it to finish; its V tile (read
// by dP only) two deep.
constexpr int K_STAGES = 3, V_STAGES = 2;
constexpr int QS_OFF = 0;                 // [Q_1; Q_2]: 2 blocks of [128 x 64]
constexpr int DO_OFF = 2 * BLK;           // [dO; dO]
constexpr int ST_OFF = 4 * BLK;           // 64 x (lse_1, lse_2, delta_1, delta_2)
constexpr int K_OFF = 4 * BLK + 1024;     // K_STAGES x K (2 blocks)
constexpr int V_OFF = K_OFF + K_STAGES * 2 * BLK;  // V_STAGES x V (2 blocks)
constexpr int MISC_OFF = V_OFF + V_STAGES * 2 * BLK;
constexpr int SMEM_BYTES = MISC_OFF + 1024 + 1024;
// TMEM columns: S, dP, dQ, dS (bf16)
constexpr int C_S = 0, C_DP = 128, C_DQ = 256, C_DS = 384;
struct Misc {
  uint64_t q_full, k_full[K_STAGES], k_empty[K_STAGES], v_full[V_STAGES], v_empty[V_STAGES];
  uint64_t s_full, p_full, o_full;
  uint64_t s_read;   // every row thread has read the step's S and dP columns
  uint64_t dq_done;  // the dQ MMAs of a step have completed (they read its dS)
  uint32_t tmem_base;
  int abort;
};
static_assert(K_OFF % 1024 == 0 && sizeof(Misc) <= 1024, "layout");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
}  // namespace dqk
}  // namespace

template <bool V1>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_v2_dq_kernel(const __grid_constant__ BwdMaps maps, const BwdArgs g) {
  using namespace dqk;
  const PrefillArgs& a = g.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + MISC_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qtiles = (a.N + QT - 1) / QT;
  const int per_qt = a.units * a.B;
  // causal: the last query tile sees the most keys, hand it out first
  const int qt = a.causal ? n_qtiles - 1 - (int)(blockIdx.x / per_qt) : (int)(blockIdx.x / per_qt);
  const int u = (int)(blockIdx.x % per_qt) % a.units;
  const int b = (int)(blockIdx.x % per_qt) / a.units;
  const int q0 = qt * QT;
  const int gk = V1 ? u : (2 * u) / a.group;
  const int off = a.Nk - a.N;
  const int khi = a.causal ? min(q0 + QT - 1 + off, a.Nk - 1) : a.Nk - 1;
  const int klo = (a.causal && a.window > 0) ? max(0, q0 + off - a.window + 1) : 0;
  const int j_lo = klo / KT;
  const int n_kt = khi >= klo ? khi / KT - j_lo + 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(&ms.q_full, 1);
    for (int s = 0; s < K_STAGES; ++s) {
      mbar_init(&ms.k_full[s], 1);
      mbar_init(&ms.k_empty[s], 1);
    }
    for (int s = 0; s < V_STAGES; ++s) {
      mbar_init(&ms.v_full[s], 1);
      mbar_init(&ms.v_empty[s], 1);
    }
    mbar_init(&ms.s_full, 1);
    mbar_init(&ms.p_full, 4 * RW);  // one arrival per row warp
    mbar_init(&ms.o_full, 1);
    mbar_init(&ms.s_read, 4 * RW);
    mbar_init(&ms.dq_done, 1);
    ms.abort = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(&ms.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (V1) {
    // the zero quadrants of the query tile: block 0 rows 64-127, block 1 rows 0-63
    for (int i = threadIdx.x; i < 2 * (HBLK / 16); i += NUM_THREADS) {
      const int o = i < HBLK / 16 ? HBLK + 16 * i : BLK + 16 * (i - HBLK / 16);
      *reinterpret_cast<uint4*>(smem + QS_OFF + o) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  volatile int* abort_flag = &ms.abort;
  const int rows = a.N + 64;

  if (warp == W_TMA) {
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      tma_prefetch_desc(&maps.dy);
      const int64_t st_off = (((int64_t)b * a.units + u) * rows + q0) * 4;  // (workspace offset)
      const bool st_ok = in_bounds((g.w_st - g.w_base) + st_off, 256, g.ext_ws, a.dev_status, a.dbg_status);
      mbar_arrive_expect_tx(&ms.q_full, (V1 ? 2 * HBLK : 2 * BLK) + 2 * BLK + (st_ok ? 1024 : 0));
      for (int hf = 0; hf < 2; ++hf) {
        if (V1) {
          tma_load_4d(smem + QS_OFF + hf * BLK + hf * HBLK, &maps.q, &ms.q_full, 64 * hf, u, q0, b);
        } else {
          tma_load_4d(smem + QS_OFF + hf * BLK, &maps.q, &ms.q_full, 64 * hf, 2 * u, q0, b);
          tma_load_4d(smem + QS_OFF + hf * BLK + 64 * 128, &maps.q, &ms.q_full, 64 * hf, 2 * u + 1, q0, b);
        }
        // dO in both halves: the branch-2 rows need dP = dO V^T as well
        tma_load_4d(smem + DO_OFF + hf * BLK, &maps.dy, &ms.q_full, 64 * hf, u, q0, b);
        tma_load_4d(smem + DO_OFF + hf * BLK + 64 * 128, &maps.dy, &ms.q_full, 64 * hf, u, q0, b);
      }
      if (st_ok) bulk_load(smem + ST_OFF, g.w_st + st_off, 1024, &ms.q_full);
      int k_issued = 0, v_issued = 0;
      for (int t = 0; t < n_kt && !*abort_flag; ++t) {
        const int kj = (j_lo + t) * KT;
        const int sk = t % K_STAGES, sv = t % V_STAGES;
        if (!mbar_wait(&ms.k_empty[sk], ((t / K_STAGES) & 1) ^ 1, abort_flag)) break;
        uint8_t* ks = smem + K_OFF + sk * 2 * BLK;
        mbar_arrive_expect_tx(&ms.k_full[sk], 2 * BLK);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_4d(ks + hf * BLK, &maps.k, &ms.k_full[sk], 64 * hf, gk, kj, b);
        k_issued = t + 1;
        if (!mbar_wait(&ms.v_empty[sv], ((t / V_STAGES) & 1) ^ 1, abort_flag)) break;
        uint8_t* vs = smem + V_OFF + sv * 2 * BLK;
        mbar_arrive_expect_tx(&ms.v_full[sv], 2 * BLK);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_4d(vs + hf * BLK, &maps.v, &ms.v_full[sv], 64 * hf, gk, kj, b);
        v_issued = t + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(&ms.q_full, 0);
        for (int t = max(0, k_issued - K_STAGES); t < k_issued; ++t)
          mbar_wait_drain(&ms.k_full[t % K_STAGES], (t / K_STAGES) & 1);
        for (int t = max(0, v_issued - V_STAGES); t < v_issued; ++t)
          mbar_wait_drain(&ms.v_full[t % V_STAGES], (t / V_STAGES) & 1);
      }
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, 128, false, true);
      const uint64_t qd = sw128_desc(smem_u32(smem + QS_OFF), 16, 1024);
      const uint64_t dd = sw128_desc(smem_u32(smem + DO_OFF), 16, 1024);
      auto issue_s_dp = [&](int t) {
        const uint64_t kd = sw128_desc(smem_u32(smem + K_OFF + (t % K_STAGES) * 2 * BLK), 16, 1024);
        const uint64_t vd = sw128_desc(smem_u32(smem + V_OFF + (t % V_STAGES) * 2 * BLK), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk >> 2) * BLK + (kk & 3) * 32;
          umma_ss(tmem + C_S, desc_at(qd, o), desc_at(kd, o), IDESC_SS, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk >> 2) * BLK + (kk & 3) * 32;
          umma_ss(tmem + C_DP, desc_at(dd, o), desc_at(vd, o), IDESC_SS, kk > 0);
        }
        tc_commit(&ms.s_full);
        tc_commit(&ms.v_empty[t % V_STAGES]);
      };
      auto issue_dq = [&](int t) {
        // K read MN-major: K index = key
        const uint64_t kmn = sw128_desc(smem_u32(smem + K_OFF + (t % K_STAGES) * 2 * BLK), BLK, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + C_DQ, tmem + C_DS + kk * 8, desc_at(kmn, kk * 2048), IDESC_ACC,
                  (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&ms.dq_done);
        tc_commit(&ms.k_empty[t % K_STAGES]);
      };
      auto kv_ready = [&](int t) {
        return mbar_wait(&ms.k_full[t % K_STAGES], (t / K_STAGES) & 1, abort_flag) &&
               mbar_wait(&ms.v_full[t % V_STAGES], (t / V_STAGES) & 1, abort_flag);
      };
      bool ok = mbar_wait(&ms.q_full, 0, abort_flag);
      if (ok && n_kt > 0) {
        ok = kv_ready(0);
        if (ok) {
          tc_fence_after();
          issue_s_dp(0);
        }
      }
      // Per step t: S, dP of step t+1 as soon as the row threads have read step t's (into
      // the same columns), then dQ of step t once its dS is written.
      for (int t = 0; t < n_kt && ok; ++t) {
        if (t + 1 < n_kt) {
          if (!(ok = mbar_wait(&ms.s_read, t & 1, abort_flag))) break;
          if (!(ok = kv_ready(t + 1))) break;
          tc_fence_after();
          issue_s_dp(t + 1);
        }
        if (!(ok = mbar_wait(&ms.p_full, t & 1, abort_flag))) break;
        tc_fence_after();
        issue_dq(t);
      }
      tc_commit(&ms.o_full);
    }
  } else {
    // ------------- per-(query, branch) arithmetic (warps 0 .. 4 RW - 1) ---------------
    // row r (TMEM lane): branch r / 64 of query q0 + r % 64 (rows 0-63 Q_1, 64-127 Q_2);
    // warpgroup wgr takes keys 32 wgr .. 32 wgr + 31 of every 128-key step
    static_assert(RW == 4, "one 32-key chunk per row warpgroup");
    const int wgr = warp >> 2;
    const int r = (warp & 3) * 32 + lane, br = r >> 6;
    const int qi = q0 + (r & 63);
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = 1.4426950408889634f * rsqrtf((float)a.d);
    const float lam = a.lambda[u];
    bool ok = mbar_wait(&ms.q_full, 0, abort_flag);
    const float4 st = reinterpret_cast<const float4*>(smem + ST_OFF)[r & 63];
    const float lse = br ? st.y : st.x, del = br ? st.w : st.z, coef = br ? -lam : 1.f;
    for (int t = 0; t < n_kt; ++t) {
      if (ok) ok = mbar_wait(&ms.s_full, t & 1, abort_flag);
      if (!(ok = __all_sync(FULL, ok))) break;
      tc_fence_after();
      const int kj0 = (j_lo + t) * KT;
      const bool full = tile_visible(a, q0, QT, kj0, KT);
      uint32_t ds[16];
      auto chunk = [&](int c, auto all_visible) {
        float sv[32], dp[32];
        tmem_ld32f(lane_addr + dqk::C_S + 32 * c, sv);
        tmem_ld32f(lane_addr + dqk::C_DP + 32 * c, dp);
        tmem_wait_ld();
        // the next step's S and dP may now overwrite these columns (one arrival per warp)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms.s_read);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float v2[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const bool vis = decltype(all_visible)::value || visible(a, qi, kj0 + 32 * c + e + x);
            const float p = vis ? ex2(sv[e + x] * sl2 - lse) : 0.f;
            v2[x] = vis ? coef * p * (dp[e + x] - del) : 0.f;
          }
          ds[e / 2] = pack_bf16(v2[0], v2[1]);
        }
      };
      if (full) chunk(wgr, std::true_type{});
      else chunk(wgr, std::false_type{});
      // dS of step t replaces that of step t - 1 once the dQ MMAs of t - 1 have read it
      if (t > 0) {
        if (ok) ok = mbar_wait(&ms.dq_done, (t - 1) & 1, abort_flag);
        if (!(ok = __all_sync(FULL, ok))) break;
        tc_fence_after();
      }
      tmem_st16(lane_addr + C_DS + 16 * wgr, ds);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.p_full);
    }
    if (ok) ok = mbar_wait(&ms.o_full, 0, abort_flag);
    ok = __all_sync(FULL, ok);
    // warp-collective TMEM loads; only the stores depend on the query being in range
    if (ok) {
      const float scale = rsqrtf((float)a.d);
      const int64_t qrow = (int64_t)b * a.N + (qi < a.N ? qi : 0);
      // V2: the 128 columns of query head 2u + br; V1: branch br's own half (columns
      // 64 br ..) of dS [K_1 | K_2], into q's [.., H, 2, d] layout
      const int64_t dq_off = V1 ? (qrow * a.units + u) * 128 + 64 * br : (qrow * a.Hq + 2 * u + br) * 128;
      const bool store = qi < a.N && in_bounds(dq_off, V1 ? 64 : 128, g.ext_dq, a.dev_status, a.dbg_status);
      float4* dq4 = reinterpret_cast<float4*>(g.dq + dq_off);
      const uint32_t col0 = C_DQ + (V1 ? 64u * br : 0u);  // br is warp-uniform
      const int c = wgr;  // this warpgroup's 32 columns (warp-uniform)
      if (c < (V1 ? 2 : 4)) {
        if (n_kt > 0) {
          tc_fence_after();
          float x[32];
          tmem_ld32f(lane_addr + col0 + 32 * c, x);
          tmem_wait_ld();
          if (store) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              dq4[(32 * c + e) / 4] = make_float4(x[e] * scale, x[e + 1] * scale,
                                                  x[e + 2] * scale, x[e + 3] * scale);
          }
        } else if (store) {
          for (int e = 0; e < 8; ++e) dq4[8 * c + e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    if (*abort_flag) {
      mbar_wait_drain(&ms.o_full, 0);
      if (lane == 0) report_status(a.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

namespace {
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
}  // namespace

// statistics rows (N + 64 per entry and unit), the dlambda shares and, for V1, the bf16 dO
size_t bwd_tc_workspace_bytes(int variant, int B, int N, int units) {
  size_t n = up256((size_t)B * units * (N + 64) * 4 * sizeof(float)) +
             up256((size_t)B * units * N * sizeof(float));
  if (variant == DIFFATTN_V1) n += up256((size_t)B * N * units * 128 * 2);
  return n;
}

namespace {

// The statistics rows of the backward from a training forward's saved outputs instead of a
// recompute: delta_2 = dy . (O_2 / l_2) and delta_1 = dy . (O_1 / l_1) with
// O_1 / l_1 = out + lambda O_2 / l_2, per (batch entry, query, pair); one warp per row, four
// columns per lane. Writes (lse_1, lse_2, delta_1, delta_2) and the dlambda share -delta_2 in
// the layout of the statistics pass.
__global__ void __launch_bounds__(256) bwd_saved_stats_kernel(BwdArgs g, const __nv_bfloat16* out,
                                                             const __nv_bfloat16* o2, const float* lse) {
  const PrefillArgs& a = g.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + warp;  // (b * N + i) * units + u
  if (r >= (int64_t)a.B * a.N * a.units) return;
  const int u = (int)(r % a.units);
  const int64_t bi = r / a.units;
  const int i = (int)(bi % a.N), b = (int)(bi / a.N);
  // out, o2 and dy share the output layout (strides a.os)
  const int64_t off = (int64_t)b * a.os[0] + (int64_t)i * a.os[1] + (int64_t)u * a.os[2] + 4 * lane;
  float e1 = 0.f, e2 = 0.f;
  if (in_bounds(off, 4, a.ext_out, a.dev_status, a.dbg_status)) {
    const uint2 wy = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(g.dy) + off);
    const uint2 wo = *reinterpret_cast<const uint2*>(out + off);
    const uint2 w2 = *reinterpret_cast<const uint2*>(o2 + off);
    const float lam = a.lambda[u];
    const uint32_t y4[2] = {wy.x, wy.y}, o4[2] = {wo.x, wo.y}, q4[2] = {w2.x, w2.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float dy = __uint_as_float(e ? (y4[h] & 0xffff0000u) : (y4[h] << 16));
        const float ov = __uint_as_float(e ? (o4[h] & 0xffff0000u) : (o4[h] << 16));
        const float o2v = __uint_as_float(e ? (q4[h] & 0xffff0000u) : (q4[h] << 16));
        e2 = fmaf(dy, o2v, e2);
        e1 = fmaf(dy, fmaf(lam, o2v, ov), e1);
      }
    }
  }
  e1 = warp_sum(e1);
  e2 = warp_sum(e2);
  if (lane == 0) {
    const int64_t unit_row = (int64_t)b * a.units + u;
    const int64_t sr = (unit_row * (a.N + 64) + i) * 4, lr = (unit_row * a.N + i) * 2;
    if (in_bounds((g.w_st - g.w_base) + sr, 4, g.ext_ws, a.dev_status, a.dbg_status) &&
        in_bounds(lr, 2, a.ext_tr_lse, a.dev_status, a.dbg_status))
      *reinterpret_cast<float4*>(g.w_st + sr) = make_float4(lse[lr], lse[lr + 1], e1, e2);
    if (in_bounds((g.w_dl - g.w_base) + unit_row * a.N + i, 1, g.ext_ws, a.dev_status, a.dbg_status))
      g.w_dl[unit_row * a.N + i] = -e2;
  }
}

// A second stream per device for the dQ kernel: the dK/dV grid (one CTA per 128 keys and KV
// head, the first key tiles of a causal problem the heaviest) ends in a partial wave, and the
// short dQ CTAs fill the SMs it leaves idle. Forked from the caller's stream and joined back
// to it with events, so the pair stays ordered with the caller's work and can be captured
// into a CUDA graph; the mutex keeps the event records of concurrent callers apart.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool failed = false;
};
std::mutex g_side_mu;
SideStream g_side[64];

// the side stream of device dev, or nullptr (then both kernels run on the caller's stream)
SideStream* side_stream(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = g_side[dev];
  if (!ss.s && !ss.failed) {
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      ss.failed = true;
      cudaGetLastError();  // the fallback below needs no side stream; clear the error
      return nullptr;
    }
  }
  return ss.failed ? nullptr : &ss;
}

// steps 2-4 of the tensor-core backward, once the statistics rows are in the workspace
cudaError_t backward_tc_kernels(const BwdArgs& g, cudaStream_t stream) {
  const PrefillArgs& a = g.f;
  const bool v1 = a.variant == DIFFATTN_V1;
  // dK/dV and dQ. V2: q [B, N, Hq, 128], k, v [B, N, Hkv, 128], dO = dy [B, N, Hq/2, 128].
  // V1: q, k, v [B, N, H, 128] ((Q_1 | Q_2), (K_1 | K_2), V), dO the bf16 workspace rows
  // [B, N, H, 128].
  BwdMaps maps;
  if (!make_map(&maps.q, a.q, 128, v1 ? a.units : a.Hq, a.N, a.B, a.qs, 64)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, 128, a.Hkv, a.Nk, a.B, a.ks, 128)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, 128, a.Hkv, a.Nk, a.B, a.vs, 128)) return cudaErrorInvalidValue;
  if (v1) {
    const int64_t ds[3] = {(int64_t)a.N * a.units * 128, (int64_t)a.units * 128, 128};
    if (!make_map(&maps.dy, g.w_do16, 128, a.units, a.N, a.B, ds, 64)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&maps.dy, g.dy, 128, a.units, a.N, a.B, g.dys, 64)) return cudaErrorInvalidValue;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const void* kv_fns[2] = {(const void*)bwd_v2_dkdv_kernel<false>, (const void*)bwd_v2_dkdv_kernel<true>};
    const void* dq_fns[2] = {(const void*)bwd_v2_dq_kernel<false>, (const void*)bwd_v2_dq_kernel<true>};
    for (int i = 0; i < 2; ++i) {
      e = cudaFuncSetAttribute(kv_fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, kv::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(dq_fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, dqk::SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    if (dev < 64) attr_set[dev] = true;
  }
  const long long kv_ctas = (long long)((a.Nk + kv::KT - 1) / kv::KT) * a.Hkv * a.B;
  const long long dq_ctas = (long long)((a.N + dqk::QT - 1) / dqk::QT) * a.units * a.B;
  if (kv_ctas > 0x7fffffffLL || dq_ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = side_stream(dev);
  cudaStream_t dq_stream = stream;
  if (ss) {
    if ((e = cudaEventRecord(ss->fork, stream)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess) return e;
    dq_stream = ss->s;
  }
  if (v1) bwd_v2_dkdv_kernel<true><<<(unsigned)kv_ctas, NUM_THREADS, kv::SMEM_BYTES, stream>>>(maps, g);
  else bwd_v2_dkdv_kernel<false><<<(unsigned)kv_ctas, NUM_THREADS, kv::SMEM_BYTES, stream>>>(maps, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (v1) bwd_v2_dq_kernel<true><<<(unsigned)dq_ctas, NUM_THREADS, dqk::SMEM_BYTES, dq_stream>>>(maps, g);
  else bwd_v2_dq_kernel<false><<<(unsigned)dq_ctas, NUM_THREADS, dqk::SMEM_BYTES, dq_stream>>>(maps, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ss) {
    if ((e = cudaEventRecord(ss->join, ss->s)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(stream, ss->join, 0)) != cudaSuccess) return e;
  }
  return launch_dlambda_reduce(g, stream);
}

void set_tc_workspace(BwdArgs& g, void* workspace) {
  const PrefillArgs& a = g.f;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const size_t st_bytes = up256((size_t)a.B * a.units * (a.N + 64) * 4 * sizeof(float));
  const size_t dl_bytes = up256((size_t)a.B * a.units * a.N * sizeof(float));
  g.w_st = reinterpret_cast<float*>(w);
  g.w_dl = reinterpret_cast<float*>(w + st_bytes);
  g.w_do = nullptr;
  g.w_do16 = a.variant == DIFFATTN_V1 ? static_cast<void*>(w + st_bytes + dl_bytes) : nullptr;
  g.w_base = g.w_st;
}

}  // namespace

cudaError_t launch_backward_tc(BwdArgs g, void* workspace, cudaStream_t stream) {
  const PrefillArgs& a = g.f;
  const bool v1 = a.variant == DIFFATTN_V1;
  if (a.cu_q || (v1 ? a.d != 64 : a.d != 128)) return cudaErrorNotSupported;
  set_tc_workspace(g, workspace);
  // 1. statistics: the forward kernel in its statistics mode
  PrefillArgs fa = a;
  fa.out = nullptr;
  fa.st_dy = g.dy;
  for (int i = 0; i < 3; ++i) fa.st_dys[i] = g.dys[i];
  fa.st = g.w_st;
  fa.st_dl = g.w_dl;
  fa.st_rows = a.N + 64;
  fa.ext_st_dy = a.ext_out;  // dy has the output's layout
  fa.ext_st = (int64_t)a.B * a.units * (a.N + 64) * 4;
  fa.ext_st_dl = (int64_t)a.B * a.units * a.N;
  fa.st_do = g.w_do16;
  fa.ext_st_do = (int64_t)a.B * a.N * a.units * 128;
  cudaError_t e = v1 ? launch_prefill_v1_stats(fa, stream) : launch_prefill_v2_stats(fa, stream);
  if (e != cudaSuccess) return e;
  return backward_tc_kernels(g, stream);
}

cudaError_t launch_backward_tc_saved(BwdArgs g, const void* out, const void* o2, const float* lse,
                                     void* workspace, cudaStream_t stream) {
  const PrefillArgs& a = g.f;
  if (a.cu_q || a.variant != DIFFATTN_V2 || a.d != 128) return cudaErrorNotSupported;
  set_tc_workspace(g, workspace);
  g.f.ext_tr_lse = (int64_t)a.B * a.units * a.N * 2;
  const long long rows = (long long)a.B * a.N * a.units;
  if ((rows + 7) / 8 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  bwd_saved_stats_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
      g, static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(o2), lse);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return backward_tc_kernels(g, stream);
}

}  // namespace diffattn
