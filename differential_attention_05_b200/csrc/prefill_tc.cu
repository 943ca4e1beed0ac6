// prefill_tc.cu -- fused differential attention prefill on the sm_100a tensor cores.
//
// What it computes, per differential unit (V1 head / V2 query-head pair) and query row i:
//   S_b = Q_b K_b^T / sqrt(d)           b = 1, 2   (V2: K_1 = K_2 = the pair's KV head)
//   A_b = softmax(S_b) over keys j <= i (causal) or all keys
//   o   = (A_1 - lambda A_2) V           V loaded once, shared by both branches
//   V1: o <- o / sqrt(mean(o^2) + eps) * (1 - lambda_init)
// ("Differential Attention (V2)", The Concept, "The difference idea" and "V1 vs V2";
//  "Attention Variants", Build It, Steps 1 and 4; Hugging Face post, "How?").
//
// Design (one CTA per 128-query tile of one unit; heaviest causal tiles launched first):
//   * The two branches are two independent 128-row MMA problems that share every K tile
//     (V2) and every V tile (V1 and V2). TMEM holds S_1, S_2, O_1, O_2 (4 x 128 columns,
//     the full 512). P_b is written back over S_b as bf16 and fed to the P.V MMA straight
//     from TMEM, so neither map ever leaves the SM.
//   * 384 threads; after launch the registers are re-split (setmaxnreg) towards the
//     softmax warpgroups. warp 8 (one lane) issues TMA tile loads (128-byte swizzle, no multicast) into a
//     2-stage K ring and a 2-stage V ring; warp 9 (one lane) allocates TMEM and issues all
//     tcgen05.mma; warps 0-3 run the online softmax of branch 1, warps 4-7 of branch 2
//     (thread t owns TMEM lane t = query row t, so row max and row sum need no shuffles).
//     The MMA issue order S_1(j+1) after P_1(j).V lets branch 1's softmax of tile j+1
//     overlap branch 2's softmax of tile j.
//   * Online softmax in the log2 domain with a lazy rescale: the running max is only
//     raised (and O_b in TMEM rescaled) when a row max grows by more than 2^8; the final
//     O_b / l_b is exact either way.
//   * Epilogue: O_1/l_1 - lambda O_2/l_2, the V1 RMSNorm (row sum of squares exchanged
//     between the two warpgroups through shared memory) and (1 - lambda_init), bf16 store.
//   * Every mbarrier wait is bounded; a timeout raises an abort flag that makes every role
//     stop issuing, waits for outstanding copies and MMAs, frees TMEM and reports
//     DIFFATTN_ERR_TIMEOUT in dev_status.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.cuh"

namespace diffattn {

namespace {
constexpr int BM = 128;                    // queries per tile
constexpr int BN = 128;                    // keys per tile
constexpr int BLK_BYTES = 128 * 128;       // one [128 rows x 64 bf16] swizzled block
constexpr int KSTAGES = 2, VSTAGES = 2;
constexpr int Q_OFF = 0;                   // Q_1 blocks at 0, 16K; Q_2 at 32K, 48K
constexpr int K_OFF = 4 * BLK_BYTES;       // 64K
constexpr int V_OFF = K_OFF + KSTAGES * 2 * BLK_BYTES;
constexpr int MISC_OFF = V_OFF + VSTAGES * 2 * BLK_BYTES;  // 192K
constexpr int SMEM_BYTES = MISC_OFF + 4096 + 1024;         // + misc + alignment slack
constexpr int NUM_THREADS = 384;           // 8 softmax warps + TMA warp + MMA warp + 2 idle
// register split after launch (168 per thread): softmax warpgroups 208, the third 88;
// 2 * 208 + 88 = 3 * 168, so the increases are exactly covered by the decrease
constexpr int REGS_SOFTMAX = 208, REGS_OTHER = 88;
constexpr int TMEM_COLS = 512;
constexpr uint32_t COL_S1 = 0, COL_S2 = 128, COL_O1 = 256, COL_O2 = 384;
constexpr float RESCALE_LOG2 = 8.0f;       // lazy-rescale threshold (factor 256)

struct Misc {
  uint64_t q_full;
  uint64_t k_full[KSTAGES], k_empty[KSTAGES];
  uint64_t v_full[VSTAGES], v_empty[VSTAGES];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full;
  uint32_t tmem_base;
  int abort;
  float l_x[2][BM];   // row sums, exchanged between the branch warpgroups
  float ss_x[2][BM];  // V1 norm: partial sums of squares
};
static_assert(sizeof(Misc) <= 4096, "misc region");
}  // namespace

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

template <int VARIANT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ TcMaps maps, const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + MISC_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile -> (q-tile, unit, batch); the largest causal tiles are handed out first
  const int n_qt = (a.N + BM - 1) / BM;
  const int per_qt = a.units * a.B;
  const int qt = a.causal ? (n_qt - 1 - (int)(blockIdx.x / per_qt)) : (int)(blockIdx.x / per_qt);
  const int u = (int)(blockIdx.x % per_qt) % a.units;
  const int b = (int)(blockIdx.x % per_qt) / a.units;
  const int q0 = qt * BM;
  const int n_kt = a.causal ? (qt + 1) : (a.N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(&ms.q_full, 1);
    for (int s = 0; s < KSTAGES; ++s) { mbar_init(&ms.k_full[s], 1); mbar_init(&ms.k_empty[s], 1); }
    for (int s = 0; s < VSTAGES; ++s) { mbar_init(&ms.v_full[s], 1); mbar_init(&ms.v_empty[s], 1); }
    for (int br = 0; br < 2; ++br) { mbar_init(&ms.s_full[br], 1); mbar_init(&ms.p_full[br], BM); }
    mbar_init(&ms.o_full, 1);
    ms.abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&ms.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  volatile int* abort_flag = &ms.abort;

  // coordinates of the Q rows / KV head of this unit in the TMA maps
  int qh1, qh2, kvh;
  if (VARIANT == DIFFATTN_V1) {
    qh1 = qh2 = u; kvh = u;
  } else {
    qh1 = 2 * u; qh2 = 2 * u + 1; kvh = (2 * u) / a.group;
  }

  if (warp >= 8) {
    // third warpgroup: gives registers to the softmax warpgroups, then TMA / MMA roles
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
  if (warp == 8) {
    // ------------------------------ TMA producer -------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      // Q: V2 -> head 2u cols [0,64),[64,128) and head 2u+1; V1 -> q1 (x=0), q2 (x=64)
      if (VARIANT == DIFFATTN_V2) {
        mbar_arrive_expect_tx(&ms.q_full, 4 * BLK_BYTES);
        tma_load_4d(smem + Q_OFF + 0 * BLK_BYTES, &maps.q, &ms.q_full, 0, qh1, q0, b);
        tma_load_4d(smem + Q_OFF + 1 * BLK_BYTES, &maps.q, &ms.q_full, 64, qh1, q0, b);
        tma_load_4d(smem + Q_OFF + 2 * BLK_BYTES, &maps.q, &ms.q_full, 0, qh2, q0, b);
        tma_load_4d(smem + Q_OFF + 3 * BLK_BYTES, &maps.q, &ms.q_full, 64, qh2, q0, b);
      } else {
        mbar_arrive_expect_tx(&ms.q_full, 2 * BLK_BYTES);
        tma_load_4d(smem + Q_OFF + 0 * BLK_BYTES, &maps.q, &ms.q_full, 0, qh1, q0, b);
        tma_load_4d(smem + Q_OFF + 2 * BLK_BYTES, &maps.q, &ms.q_full, 64, qh1, q0, b);
      }
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kt && !*abort_flag; ++j) {
        const int ks = j % KSTAGES, vs = j % VSTAGES;
        if (!mbar_wait(&ms.k_empty[ks], ((j / KSTAGES) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&ms.k_full[ks], 2 * BLK_BYTES);
        uint8_t* kd = smem + K_OFF + ks * 2 * BLK_BYTES;
        tma_load_4d(kd, &maps.k, &ms.k_full[ks], 0, kvh, j * BN, b);
        tma_load_4d(kd + BLK_BYTES, &maps.k, &ms.k_full[ks], 64, kvh, j * BN, b);
        ++issued_k;
        if (!mbar_wait(&ms.v_empty[vs], ((j / VSTAGES) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&ms.v_full[vs], 2 * BLK_BYTES);
        uint8_t* vd = smem + V_OFF + vs * 2 * BLK_BYTES;
        tma_load_4d(vd, &maps.v, &ms.v_full[vs], 0, kvh, j * BN, b);
        tma_load_4d(vd + BLK_BYTES, &maps.v, &ms.v_full[vs], 64, kvh, j * BN, b);
        ++issued_v;
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA's shared memory goes away
        mbar_wait_drain(&ms.q_full, 0);
        for (int j = max(0, issued_k - KSTAGES); j < issued_k; ++j)
          mbar_wait_drain(&ms.k_full[j % KSTAGES], (j / KSTAGES) & 1);
        for (int j = max(0, issued_v - VSTAGES); j < issued_v; ++j)
          mbar_wait_drain(&ms.v_full[j % VSTAGES], (j / VSTAGES) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------ MMA issuer ---------------------------------------
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, 128, false, true);
      const uint32_t qbase = smem_u32(smem + Q_OFF);
      const uint32_t kbase = smem_u32(smem + K_OFF);
      const uint32_t vbase = smem_u32(smem + V_OFF);
      bool ok = mbar_wait(&ms.q_full, 0, abort_flag);
      tc_fence_after();

      // S_br(j) = Q_br K_br(j)^T into TMEM columns of S_br
      auto issue_s = [&](int br, int j) {
        const uint32_t kst = kbase + (j % KSTAGES) * 2 * BLK_BYTES;
        const uint32_t qb = qbase + br * 2 * BLK_BYTES;
        const uint32_t dcol = tmem + (br ? COL_S2 : COL_S1);
        if (VARIANT == DIFFATTN_V2) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * BLK_BYTES + (kk & 3) * 32;
            umma_ss(dcol, sw128_desc(qb + off, 16, 1024), sw128_desc(kst + off, 16, 1024),
                    IDESC_S, kk > 0);
          }
        } else {
          const uint32_t kb = kst + br * BLK_BYTES;  // K_1 block / K_2 block
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            umma_ss(dcol, sw128_desc(qb + kk * 32, 16, 1024), sw128_desc(kb + kk * 32, 16, 1024),
                    IDESC_S, kk > 0);
          }
        }
        tc_commit(&ms.s_full[br]);
      };
      // O_br += P_br(j) V(j); P_br read from TMEM (bf16 over the S_br columns)
      auto issue_pv = [&](int br, int j) {
        const uint32_t vst = vbase + (j % VSTAGES) * 2 * BLK_BYTES;
        const uint32_t pcol = tmem + (br ? COL_S2 : COL_S1);
        const uint32_t dcol = tmem + (br ? COL_O2 : COL_O1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // MN-major B: keys step 16 rows (2048 B); the two 64-column blocks are 16 KB apart
          umma_ts(dcol, pcol + kk * 8, sw128_desc(vst + kk * 2048, BLK_BYTES, 1024), IDESC_PV,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
      };

      if (ok) ok = mbar_wait(&ms.k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        tc_commit(&ms.k_empty[0]);
      }
      for (int j = 0; j < n_kt && ok; ++j) {
        const int vs = j % VSTAGES;
        if (!(ok = mbar_wait(&ms.v_full[vs], (j / VSTAGES) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&ms.p_full[0], j & 1, abort_flag))) break;
        tc_fence_after();
        issue_pv(0, j);
        const bool more = j + 1 < n_kt;
        if (more) {
          const int ks = (j + 1) % KSTAGES;
          if (!(ok = mbar_wait(&ms.k_full[ks], ((j + 1) / KSTAGES) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (!(ok = mbar_wait(&ms.p_full[1], j & 1, abort_flag))) break;
        tc_fence_after();
        issue_pv(1, j);
        tc_commit(&ms.v_empty[vs]);
        if (more) {
          issue_s(1, j + 1);
          tc_commit(&ms.k_empty[(j + 1) % KSTAGES]);
        }
      }
      tc_commit(&ms.o_full);  // arrives once every MMA issued above has completed
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // ------------------------- softmax warpgroups (branch br) -------------------------
    const int br = warp >> 2;              // 0: warps 0-3, 1: warps 4-7
    const int row = (warp & 3) * 32 + lane;  // TMEM lane == query row in the tile
    const int qi = q0 + row;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = lane_addr + (br ? COL_S2 : COL_S1);
    const uint32_t o_col = lane_addr + (br ? COL_O2 : COL_O1);
    const float sl2 = 1.4426950408889634f * rsqrtf((float)a.d);  // log2(e)/sqrt(d)
    float m = -INFINITY, l = 0.f;
    bool ok = true;

    for (int j = 0; j < n_kt; ++j) {
      ok = mbar_wait(&ms.s_full[br], j & 1, abort_flag);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;  // tcgen05.ld/st below are warp-wide
      tc_fence_after();
      // S row (raw scores) -> registers: four loads in flight, one wait
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32f(s_col + c * 32, s + c * 32);
      tmem_wait_ld();
      // mask: causal diagonal tile, or keys past N when not causal
      const int k0 = j * BN;
      const int lim = a.causal ? (qi - k0) : (a.N - 1 - k0);  // last visible key offset
      if (lim < BN - 1) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e > lim) s[e] = -INFINITY;
      }
      // row max: four independent chains of 3-input max
      float c0 = -INFINITY, c1 = -INFINITY, c2 = -INFINITY, c3 = -INFINITY;
#pragma unroll
      for (int e = 0; e < BN; e += 8) {
        c0 = fmax3(c0, s[e + 0], s[e + 1]);
        c1 = fmax3(c1, s[e + 2], s[e + 3]);
        c2 = fmax3(c2, s[e + 4], s[e + 5]);
        c3 = fmax3(c3, s[e + 6], s[e + 7]);
      }
      const float mx = fmax3(fmaxf(c0, c1), c2, c3) * sl2;  // log2 domain
      // raise the running max only when it grew by more than 2^8 (or was unset); the
      // decision is per row, the O rescale below is done by the whole warp when any of
      // its rows needs it (rows that do not use alpha = 1)
      const bool raise = (mx > m + RESCALE_LOG2) || (m == -INFINITY);
      const float mn = raise ? fmaxf(mx, m) : m;
      const float alpha = (raise && m != -INFINITY) ? ex2(m - mn) : 1.f;
      if (__any_sync(0xffffffffu, raise && m != -INFINITY)) {
        // O_br row *= alpha (its last P.V MMA completed before S_br(j) did)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(o_col + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(o_col + c * 32, r);
        }
      }
      l *= alpha;
      m = mn;
      // P = 2^(s * log2(e)/sqrt(d) - m), summed in fp32, stored as bf16 over S_br
      const float nm = (m == -INFINITY) ? 0.f : -m;  // fully masked row: all p = 0
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, a4 = 0.f, a5 = 0.f, a6 = 0.f, a7 = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float x0, x1, x2, x3;
          ffma2(x0, x1, s[c * 64 + 2 * e], s[c * 64 + 2 * e + 1], sl2, sl2, nm, nm);
          ffma2(x2, x3, s[c * 64 + 2 * e + 2], s[c * 64 + 2 * e + 3], sl2, sl2, nm, nm);
          const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
          if ((e & 2) == 0) {
            fadd2(a0, a1, a0, a1, p0, p1);
            fadd2(a2, a3, a2, a3, p2, p3);
          } else {
            fadd2(a4, a5, a4, a5, p0, p1);
            fadd2(a6, a7, a6, a7, p2, p3);
          }
          pk[e] = pack_bf16(p0, p1);
          pk[e + 1] = pack_bf16(p2, p3);
        }
        tmem_st32(s_col + c * 32, pk);
      }
      const float ps = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
      l += ps;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ms.p_full[br]);
    }

    // ------------------------------- epilogue ----------------------------------------
    if (ok) ok = mbar_wait(&ms.o_full, 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    ms.l_x[br][row] = l;
    named_bar_sync(1, 256);
    if (ok) {
      tc_fence_after();
      const float inv1 = 1.f / ms.l_x[0][row], inv2 = 1.f / ms.l_x[1][row];
      const float lam = a.lambda[u];
      // this warpgroup finishes output columns [64 br, 64 br + 64)
      float y[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r1[32], r2[32];
        tmem_ld32(lane_addr + COL_O1 + br * 64 + c * 32, r1);
        tmem_ld32(lane_addr + COL_O2 + br * 64 + c * 32, r2);
        tmem_wait_ld();
        // a_b = O_b / l_b rounded on its own, then one fused a_1 - lambda a_2: identical
        // branches with lambda = 1 give exactly 0 (no contraction across the subtraction)
#pragma unroll
        for (int e = 0; e < 32; ++e)
          y[c * 32 + e] = __fmaf_rn(-lam, __fmul_rn(__uint_as_float(r2[e]), inv2),
                                    __fmul_rn(__uint_as_float(r1[e]), inv1));
      }
      if (VARIANT == DIFFATTN_V1 && a.apply_norm) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) ss = fmaf(y[e], y[e], ss);
        ms.ss_x[br][row] = ss;
        named_bar_sync(1, 256);
        const float tot = ms.ss_x[0][row] + ms.ss_x[1][row];
        const float sc = rsqrtf(tot * (1.f / 128.f) + a.eps) * (1.f - a.lambda_init[0]);
#pragma unroll
        for (int e = 0; e < 64; ++e) y[e] *= sc;
      }
      if (qi < a.N) {
        __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.out) + (int64_t)b * a.os[0] +
                            (int64_t)qi * a.os[1] + (int64_t)u * a.os[2] + br * 64;
        uint4* o4 = reinterpret_cast<uint4*>(ob);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 w;
          w.x = pack_bf16(y[v * 8 + 0], y[v * 8 + 1]);
          w.y = pack_bf16(y[v * 8 + 2], y[v * 8 + 3]);
          w.z = pack_bf16(y[v * 8 + 4], y[v * 8 + 5]);
          w.w = pack_bf16(y[v * 8 + 6], y[v * 8 + 7]);
          o4[v] = w;
        }
      }
    } else if (VARIANT == DIFFATTN_V1 && a.apply_norm) {
      named_bar_sync(1, 256);  // keep the barrier count of the normal path
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    if (*abort_flag) {
      // wait (bounded) for any MMA still in flight before giving TMEM back
      mbar_wait_drain(&ms.o_full, 0);
      if (threadIdx.x == 9 * 32) report_status(a.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------
// host side

namespace {

template <int VARIANT>
cudaError_t launch_variant(const PrefillArgs& a, cudaStream_t stream) {
  TcMaps maps;
  const int C = 128;  // V1: [q1|q2] / [k1|k2] / v of width 2d = 128; V2: d = 128
  const int hq = VARIANT == DIFFATTN_V1 ? a.units : a.Hq;
  const int hkv = VARIANT == DIFFATTN_V1 ? a.units : a.Hkv;
  if (!make_map(&maps.q, a.q, C, hq, a.N, a.B, a.qs)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, C, hkv, a.N, a.B, a.ks)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, C, hkv, a.N, a.B, a.vs)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(prefill_tc_kernel<VARIANT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  const long long tiles = (long long)((a.N + BM - 1) / BM) * a.units * a.B;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  prefill_tc_kernel<VARIANT><<<(unsigned)tiles, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream) {
  if (a.variant == DIFFATTN_V1) {
    if (a.d != 64) return cudaErrorNotSupported;
    return launch_prefill_tc_v1(a, stream);  // two-pass kernel (prefill_tc_v1.cu)
  }
  if (a.d != 128 || a.group % 2 != 0) return cudaErrorNotSupported;
  return launch_variant<DIFFATTN_V2>(a, stream);
}

}  // namespace diffattn
