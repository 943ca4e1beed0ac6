// prefill_tc_v1.cu -- V1 differential attention prefill on the sm_100a tensor cores, with
// the per-head RMSNorm and (1 - lambda_init) scale fused into the epilogue.
//
// V1 ("Differential Attention (V2)", "V1 vs V2"): each head splits Q, K into two branches of
// width d = 64 with separate K_1, K_2, and one V of width 2d = 128 shared by both branches;
// after the difference comes a per-head RMSNorm, then the (1 - lambda_init) factor.
//
// Why two passes. The V1 workload feeds 1/sqrt(d)-scaled inputs, so both maps are close to
// uniform and A_1 - lambda A_2 is much smaller than either map when lambda nears 1. Rounding
// each branch's probabilities to bf16 (the MMA operand type) before the subtraction puts a
// relative error of 2^-9 on A_1 and A_2 separately, which the difference amplifies by about
// 1/(1 - lambda) and the RMSNorm then scales up to unit size. So the weights are formed
// exactly first and rounded once:
//   pass 1: S_b = Q_b K_b^T for every key tile, b = 1, 2; per row, the running max m_b and
//           sum l_b of 2^(S_b log2(e)/sqrt(d) - m_b)  (no P.V)
//   pass 2: S_b again; W = 2^(S_1.. - m_1)/l_1 - lambda 2^(S_2.. - m_2)/l_2 in fp32, rounded
//           to bf16 once, and a single MMA O += W V per key tile
//   epilogue: O / sqrt(mean(O^2) + eps) * (1 - lambda_init), bf16 store
// The tensor-core work equals the single-pass form for V1 (QK^T twice at width 64, P.V once
// at width 128 instead of twice); the exponentials double.
//
// Roles (384 threads, registers re-split after launch): warps 0-3 own branch 1, warps 4-7
// branch 2 (thread t = TMEM lane t = query row t); warp 8 issues TMA loads (no multicast),
// warp 9 allocates TMEM and issues every tcgen05.mma. Pass 1 double-buffers both S tiles
// (4 x 128 TMEM columns). In pass 2, TMEM holds S_1, S_2, T_2 (branch 2's fp32 term
// lambda p_2 / l_2, handed to branch 1) and O; branch 2 runs one key tile ahead of branch 1.
// Every wait is bounded (see common.cuh); a timeout raises the abort flag, drains the copies
// and MMAs in flight, frees TMEM and reports DIFFATTN_ERR_TIMEOUT in dev_status.
#include "common.cuh"
#include "kernels.h"
#include "tma_host.cuh"

namespace diffattn {

namespace {
constexpr int BM = 128;                       // queries per tile
constexpr int BN = 128;                       // keys per tile
constexpr int BLK = 128 * 128;                // one [128 rows x 64 bf16] swizzled block
constexpr int KSTAGES = 3, VSTAGES = 2;
constexpr int Q_OFF = 0;                      // Q_1 block at 0, Q_2 block at 16K
constexpr int K_OFF = 2 * BLK;                // each K stage: K_1 block + K_2 block
constexpr int V_OFF = K_OFF + KSTAGES * 2 * BLK;
constexpr int MISC_OFF = V_OFF + VSTAGES * 2 * BLK;
constexpr int SMEM_BYTES = MISC_OFF + 4096 + 1024;
constexpr int NUM_THREADS = 384;
constexpr int REGS_SOFTMAX = 208, REGS_OTHER = 88;  // 2 * 208 + 88 = 3 * 168
constexpr int TMEM_COLS = 512;
// pass 1: S of branch br, buffer f at column 128 * br + 256 * f
__host__ __device__ constexpr uint32_t p1_col(int br, int f) { return 128u * br + 256u * f; }
constexpr uint32_t COL_S1 = 0, COL_S2 = 128, COL_T2 = 256, COL_O = 384;  // pass 2
constexpr float RESCALE_LOG2 = 8.0f;

struct Misc {
  uint64_t q_full;
  uint64_t k_full[KSTAGES], k_empty[KSTAGES];
  uint64_t v_full[VSTAGES], v_empty[VSTAGES];
  uint64_t s_full[2][2], s_free[2][2];  // pass 1, [branch][buffer]
  uint64_t pass1_done;                  // every softmax thread has finished pass 1
  uint64_t s1_full, s2_full, s2_free, t2_full, t2_free, p_full, o_full;  // pass 2
  uint32_t tmem_base;
  int abort;
  float ss_x[2][BM];
};
static_assert(sizeof(Misc) <= 4096, "misc region");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
}  // namespace

__device__ __forceinline__ void bar_sync_softmax() {
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_tc_v1_kernel(const __grid_constant__ TcMaps maps, const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + MISC_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int n_qt = (a.N + BM - 1) / BM;
  const int per_qt = a.units * a.B;
  const int qt = a.causal ? (n_qt - 1 - (int)(blockIdx.x / per_qt)) : (int)(blockIdx.x / per_qt);
  const int u = (int)(blockIdx.x % per_qt) % a.units;  // head
  const int b = (int)(blockIdx.x % per_qt) / a.units;
  const int q0 = qt * BM;
  const int n_kt = a.causal ? (qt + 1) : (a.N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(&ms.q_full, 1);
    for (int s = 0; s < KSTAGES; ++s) { mbar_init(&ms.k_full[s], 1); mbar_init(&ms.k_empty[s], 1); }
    for (int s = 0; s < VSTAGES; ++s) { mbar_init(&ms.v_full[s], 1); mbar_init(&ms.v_empty[s], 1); }
    for (int br = 0; br < 2; ++br)
      for (int f = 0; f < 2; ++f) { mbar_init(&ms.s_full[br][f], 1); mbar_init(&ms.s_free[br][f], BM); }
    mbar_init(&ms.pass1_done, 2 * BM);
    mbar_init(&ms.s1_full, 1);
    mbar_init(&ms.s2_full, 1);
    mbar_init(&ms.s2_free, BM);
    mbar_init(&ms.t2_full, BM);
    mbar_init(&ms.t2_free, BM);
    mbar_init(&ms.p_full, BM);
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

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
    if (warp == 8 && lane == 0) {
      // ------------------------------ TMA producer -----------------------------------
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      mbar_arrive_expect_tx(&ms.q_full, 2 * BLK);
      tma_load_4d(smem + Q_OFF, &maps.q, &ms.q_full, 0, u, q0, b);         // q_1
      tma_load_4d(smem + Q_OFF + BLK, &maps.q, &ms.q_full, 64, u, q0, b);  // q_2
      int issued_k = 0, issued_v = 0;
      // K tiles 0..n-1 for pass 1, then K and V tiles 0..n-1 for pass 2
      for (int t = 0; t < 2 * n_kt && !*abort_flag; ++t) {
        const int j = t < n_kt ? t : t - n_kt;
        const int ks = t % KSTAGES;
        if (!mbar_wait(&ms.k_empty[ks], ((t / KSTAGES) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&ms.k_full[ks], 2 * BLK);
        uint8_t* kd = smem + K_OFF + ks * 2 * BLK;
        tma_load_4d(kd, &maps.k, &ms.k_full[ks], 0, u, j * BN, b);         // k_1
        tma_load_4d(kd + BLK, &maps.k, &ms.k_full[ks], 64, u, j * BN, b);  // k_2
        ++issued_k;
        if (t >= n_kt) {
          const int vs = j % VSTAGES;
          if (!mbar_wait(&ms.v_empty[vs], ((j / VSTAGES) & 1) ^ 1, abort_flag)) break;
          mbar_arrive_expect_tx(&ms.v_full[vs], 2 * BLK);
          uint8_t* vd = smem + V_OFF + vs * 2 * BLK;
          tma_load_4d(vd, &maps.v, &ms.v_full[vs], 0, u, j * BN, b);
          tma_load_4d(vd + BLK, &maps.v, &ms.v_full[vs], 64, u, j * BN, b);
          ++issued_v;
        }
      }
      if (*abort_flag) {
        mbar_wait_drain(&ms.q_full, 0);
        for (int t = max(0, issued_k - KSTAGES); t < issued_k; ++t)
          mbar_wait_drain(&ms.k_full[t % KSTAGES], (t / KSTAGES) & 1);
        for (int j = max(0, issued_v - VSTAGES); j < issued_v; ++j)
          mbar_wait_drain(&ms.v_full[j % VSTAGES], (j / VSTAGES) & 1);
      }
    } else if (warp == 9 && lane == 0) {
      // ------------------------------ MMA issuer -------------------------------------
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, 128, false, true);
      const uint32_t qbase = smem_u32(smem + Q_OFF);
      const uint32_t kbase = smem_u32(smem + K_OFF);
      const uint32_t vbase = smem_u32(smem + V_OFF);
      // S_br = Q_br K_br^T from K load t (stage t % KSTAGES) into TMEM column dcol
      auto issue_s = [&](uint32_t dcol, int br, int t) {
        const uint32_t qb = qbase + br * BLK;
        const uint32_t kb = kbase + (t % KSTAGES) * 2 * BLK + br * BLK;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tmem + dcol, sw128_desc(qb + kk * 32, 16, 1024), sw128_desc(kb + kk * 32, 16, 1024),
                  IDESC_S, kk > 0);
      };
      bool ok = mbar_wait(&ms.q_full, 0, abort_flag);
      // pass 1
      for (int j = 0; j < n_kt && ok; ++j) {
        const int f = j & 1, use = j >> 1;
        if (!(ok = mbar_wait(&ms.k_full[j % KSTAGES], (j / KSTAGES) & 1, abort_flag))) break;
        for (int br = 0; br < 2 && ok; ++br) {
          if (!(ok = mbar_wait(&ms.s_free[br][f], (use & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          issue_s(p1_col(br, f), br, j);
          tc_commit(&ms.s_full[br][f]);
        }
        if (ok) tc_commit(&ms.k_empty[j % KSTAGES]);
      }
      // pass 2 starts once both warpgroups have read their last pass-1 scores
      if (ok) ok = mbar_wait(&ms.pass1_done, 0, abort_flag);
      if (ok) ok = mbar_wait(&ms.k_full[n_kt % KSTAGES], (n_kt / KSTAGES) & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(COL_S1, 0, n_kt);
        tc_commit(&ms.s1_full);
        issue_s(COL_S2, 1, n_kt);
        tc_commit(&ms.s2_full);
        tc_commit(&ms.k_empty[n_kt % KSTAGES]);
      }
      for (int j = 0; j < n_kt && ok; ++j) {
        const bool more = j + 1 < n_kt;
        const int t1 = n_kt + j + 1;
        if (more) {
          if (!(ok = mbar_wait(&ms.k_full[t1 % KSTAGES], (t1 / KSTAGES) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&ms.s2_free, j & 1, abort_flag))) break;
          tc_fence_after();
          issue_s(COL_S2, 1, t1);  // branch 2 runs one tile ahead
          tc_commit(&ms.s2_full);
        }
        const int vs = j % VSTAGES;
        if (!(ok = mbar_wait(&ms.v_full[vs], (j / VSTAGES) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&ms.p_full, j & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t vst = vbase + vs * 2 * BLK;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // O += W V: W (bf16) over the S_1 columns
          umma_ts(tmem + COL_O, tmem + COL_S1 + kk * 8, sw128_desc(vst + kk * 2048, BLK, 1024),
                  IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&ms.v_empty[vs]);
        if (more) {
          issue_s(COL_S1, 0, t1);
          tc_commit(&ms.s1_full);
          tc_commit(&ms.k_empty[t1 % KSTAGES]);
        }
      }
      tc_commit(&ms.o_full);  // arrives once every MMA issued above has completed
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // --------------------------- softmax warpgroups ------------------------------------
    const int br = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int qi = q0 + row;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = 1.4426950408889634f * rsqrtf((float)a.d);  // log2(e)/sqrt(d)
    float m = -INFINITY, l = 0.f;
    bool ok = true;

    // ---- pass 1: row statistics of this branch ----
    for (int j = 0; j < n_kt; ++j) {
      const int f = j & 1;
      ok = mbar_wait(&ms.s_full[br][f], (j >> 1) & 1, abort_flag);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32f(lane_addr + p1_col(br, f) + c * 32, s + c * 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ms.s_free[br][f]);
      const int k0 = j * BN;
      const int lim = a.causal ? (qi - k0) : (a.N - 1 - k0);  // last visible key offset
      if (lim < BN - 1) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e > lim) s[e] = -INFINITY;
      }
      float c0 = -INFINITY, c1 = -INFINITY, c2 = -INFINITY, c3 = -INFINITY;
#pragma unroll
      for (int e = 0; e < BN; e += 8) {
        c0 = fmax3(c0, s[e + 0], s[e + 1]);
        c1 = fmax3(c1, s[e + 2], s[e + 3]);
        c2 = fmax3(c2, s[e + 4], s[e + 5]);
        c3 = fmax3(c3, s[e + 6], s[e + 7]);
      }
      const float mx = fmax3(fmaxf(c0, c1), c2, c3) * sl2;
      if (mx > m + RESCALE_LOG2 || m == -INFINITY) {
        const float mn = fmaxf(mx, m);
        if (m != -INFINITY) l *= ex2(m - mn);
        m = mn;
      }
      const float nm = (m == -INFINITY) ? 0.f : -m;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, a4 = 0.f, a5 = 0.f, a6 = 0.f, a7 = 0.f;
#pragma unroll
      for (int e = 0; e < BN; e += 8) {
        float x[8];
        ffma2(x[0], x[1], s[e + 0], s[e + 1], sl2, sl2, nm, nm);
        ffma2(x[2], x[3], s[e + 2], s[e + 3], sl2, sl2, nm, nm);
        ffma2(x[4], x[5], s[e + 4], s[e + 5], sl2, sl2, nm, nm);
        ffma2(x[6], x[7], s[e + 6], s[e + 7], sl2, sl2, nm, nm);
        fadd2(a0, a1, a0, a1, ex2(x[0]), ex2(x[1]));
        fadd2(a2, a3, a2, a3, ex2(x[2]), ex2(x[3]));
        fadd2(a4, a5, a4, a5, ex2(x[4]), ex2(x[5]));
        fadd2(a6, a7, a6, a7, ex2(x[6]), ex2(x[7]));
      }
      l += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
    }
    // both warpgroups finish pass 1 before pass 2 reuses the pass-1 TMEM columns
    tc_fence_before();
    mbar_arrive(&ms.pass1_done);
    if (ok) ok = mbar_wait(&ms.pass1_done, 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);

    // ---- pass 2: exact differential weights, rounded once ----
    // 2^(x sl2 - m) / l = 2^(x sl2 + off) with off = -m - log2(l) (branch 2 also folds |lambda|)
    const float lam = a.lambda[u];
    float off = -m - log2f(l);
    if (br == 1) off += log2f(fabsf(lam));  // lambda = 0: off = -inf, the term vanishes
    for (int j = 0; j < n_kt && ok; ++j) {
      const int k0 = j * BN;
      const int lim = a.causal ? (qi - k0) : (a.N - 1 - k0);
      float s[BN];
      if (br == 1) {
        ok = mbar_wait(&ms.s2_full, j & 1, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32f(lane_addr + COL_S2 + c * 32, s + c * 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&ms.s2_free);
        if (lim < BN - 1) {
#pragma unroll
          for (int e = 0; e < BN; ++e)
            if (e > lim) s[e] = -INFINITY;
        }
#pragma unroll
        for (int e = 0; e < BN; e += 2) {
          float x0, x1;
          ffma2(x0, x1, s[e], s[e + 1], sl2, sl2, off, off);
          s[e] = ex2(x0);
          s[e + 1] = ex2(x1);
        }
        ok = mbar_wait(&ms.t2_free, (j & 1) ^ 1, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(s[c * 32 + e]);
          tmem_st32(lane_addr + COL_T2 + c * 32, r);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ms.t2_full);
      } else {
        ok = mbar_wait(&ms.s1_full, j & 1, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32f(lane_addr + COL_S1 + c * 32, s + c * 32);
        tmem_wait_ld();
        if (lim < BN - 1) {
#pragma unroll
          for (int e = 0; e < BN; ++e)
            if (e > lim) s[e] = -INFINITY;
        }
#pragma unroll
        for (int e = 0; e < BN; e += 2) {
          float x0, x1;
          ffma2(x0, x1, s[e], s[e + 1], sl2, sl2, off, off);
          s[e] = ex2(x0);
          s[e + 1] = ex2(x1);
        }
        ok = mbar_wait(&ms.t2_full, j & 1, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        const float ng = lam < 0.f ? 1.f : -1.f;  // W = p_1 - sign(lambda) t_2
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          float t[32];
          tmem_ld32f(lane_addr + COL_T2 + c * 32, t);
          tmem_wait_ld();
          if (c == BN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&ms.t2_free);
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float w0, w1;
            ffma2(w0, w1, t[e], t[e + 1], ng, ng, s[c * 32 + e], s[c * 32 + e + 1]);
            pk[e / 2] = pack_bf16(w0, w1);
          }
          tmem_st16(lane_addr + COL_S1 + c * 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ms.p_full);
      }
    }

    // ---- epilogue: RMSNorm over the 2d = 128 channels, (1 - lambda_init), bf16 ----
    if (ok) ok = mbar_wait(&ms.o_full, 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    float y[64];
    float ss = 0.f;
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) tmem_ld32f(lane_addr + COL_O + br * 64 + c * 32, y + c * 32);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 64; ++e) ss = fmaf(y[e], y[e], ss);
    }
    ms.ss_x[br][row] = ss;
    bar_sync_softmax();
    if (ok) {
      float sc = 1.f;
      if (a.apply_norm) {
        const float tot = ms.ss_x[0][row] + ms.ss_x[1][row];
        sc = rsqrtf(tot * (1.f / 128.f) + a.eps) * (1.f - a.lambda_init[0]);
      }
      if (qi < a.N) {
        __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.out) + (int64_t)b * a.os[0] +
                            (int64_t)qi * a.os[1] + (int64_t)u * a.os[2] + br * 64;
        uint4* o4 = reinterpret_cast<uint4*>(ob);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 w;
          w.x = pack_bf16(y[v * 8 + 0] * sc, y[v * 8 + 1] * sc);
          w.y = pack_bf16(y[v * 8 + 2] * sc, y[v * 8 + 3] * sc);
          w.z = pack_bf16(y[v * 8 + 4] * sc, y[v * 8 + 5] * sc);
          w.w = pack_bf16(y[v * 8 + 6] * sc, y[v * 8 + 7] * sc);
          o4[v] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    if (*abort_flag) {
      mbar_wait_drain(&ms.o_full, 0);
      if (lane == 0) report_status(a.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_prefill_tc_v1(const PrefillArgs& a, cudaStream_t stream) {
  TcMaps maps;
  // q, k viewed as [B, N, H, 128] (branch 1 in columns 0..63, branch 2 in 64..127); v is 2d wide
  if (!make_map(&maps.q, a.q, 128, a.units, a.N, a.B, a.qs)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, 128, a.units, a.N, a.B, a.ks)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, 128, a.units, a.N, a.B, a.vs)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(prefill_tc_v1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  const long long tiles = (long long)((a.N + BM - 1) / BM) * a.units * a.B;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  prefill_tc_v1_kernel<<<(unsigned)tiles, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace diffattn
