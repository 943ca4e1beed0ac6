// prefill_v2.cu -- single-pass fused differential attention prefill on the sm_100a tensor
// cores, V2 (query-head pairs sharing a KV head, d = 128). V1 runs on prefill_v1.cu.
//
// What it computes, per query-head pair (2u, 2u+1) and query row i:
//   A_b = softmax(Q_b K^T / sqrt(d)) over keys j <= i (causal) or all keys,  b = 1, 2
//   o   = (A_1 - lambda A_2) V          (K, V of the pair's KV head)
// ("Differential Attention (V2)", The Concept, "The difference idea" and "V1 vs V2";
//  "Attention Variants", Build It, Steps 1 and 4).
//
// Precision. Rounding the two branches' probabilities to bf16 separately and subtracting
// afterwards loses the difference when the branches nearly cancel (lambda near 1, similar
// maps): the 2^-9 rounding error of each map is amplified by about 1/(1 - lambda). So the
// kernel accumulates, per query,
//   D   = sum_j (p1_j - c p2_j) v_j      with c near lambda l_1 / l_2
//   O_2 = sum_j p2_j v_j
// where p_b = 2^(s_b log2(e)/sqrt(d) - m_b) and m_b is branch b's running maximum. The
// operand p1 - c p2 is formed in fp32 from the exact p1, p2 and rounded once, so it carries
// an error relative to the (small) difference itself. At the end
//   o = O_1/l_1 - lambda O_2/l_2 = D/l_1 + O_2 (c/l_1 - lambda/l_2),
// and the rounding error of O_2 enters only through c/l_1 - lambda/l_2, which is small as
// c tracks lambda l_1 / l_2. D = O_1 - c O_2 is kept exact across updates: raising m_1
// (factor a_1) or m_2 (factor a_2) and moving c to c' maps D -> a_1 D + (a_1 c - a_2 c') O_2
// and O_2 -> a_2 O_2. With c' = c a_1 / a_2 the cross term vanishes; c is reset to its
// target (cross term included) only when it leaves [0.8, 1.25] times the target. Maxima are
// raised lazily, only when they grow by more than 2^8.
//
// Tensor-core shape. A tcgen05.mma costs about the same time for any N up to 128, so the
// products run at M = 128, N = 128: both branches share K, so one score MMA covers 64
// queries x both branches x 128 keys, and one P.V MMA 64 queries x both branches x 128 value
// columns (half the score instructions of a layout with a row per query and 64-key tiles).
//   * TMEM lane / operand row of (query t, branch b) in a 64-query sub-tile:
//     (t % 16) + 32 (t / 16) + 16 b; the Q rows are loaded in this order (16-row boxes
//     alternating the two heads of the pair).
//   * Warp w of a softmax warpgroup owns queries 16w..16w+15; lane l takes query 16w + l % 16
//     and half l / 16 of the key tile (64 keys) and of the value columns. The split 16-lane
//     TMEM loads give it both branches' scores of its keys (the branch-1 row and the branch-2
//     row 16 lanes further on), so p1 - c p2 is formed in registers; the two halves of a
//     query exchange only their maxima and sums. It writes the bf16 P rows of both branches
//     (p1 - c p2 over the branch-1 row, p2 over the branch-2 row); the P.V MMA (A = P from
//     TMEM) leaves D in the branch-1 lanes and O_2 in the branch-2 lanes.
//   * CTA order: bands of 32 query tiles, heaviest causal band first; inside a band KV group
//     by KV group, so the CTAs in flight read the K/V of one or two KV heads, which stay in
//     L2.
//   * Two 64-query sub-tiles per CTA (128 queries share every K/V tile) ping-pong: while
//     one warpgroup turns its scores into P, the tensor core runs the other sub-tile's
//     products. TMEM: S/P of sub-tile 0 | O of sub-tile 0 | S/P of 1 | O of 1 (4 x 128
//     columns). P (bf16) overwrites the first 64 columns of its S block; the next score
//     MMA of that sub-tile is issued after its P.V MMA, and tcgen05 MMAs run in order.
//   * Exponentials: in every 8 keys one pair is evaluated on the FMA pipe (exp2_fma2), the
//     rest on the MUFU unit; launches long enough to run under the power cap use MUFU only.
//   * warp 8: TMA loads (128-byte swizzle, no multicast) of Q once and of K, V per 128-key
//     tile into 2-stage rings; warp 9: TMEM allocation and every tcgen05.mma / commit.
//     Registers are re-split after launch (setmaxnreg): 200 for the softmax warpgroups, 104
//     for the third; 2 * 200 + 104 = 3 * 168, the launch allocation.
//   * every mbarrier wait is bounded; a timeout raises an abort flag so every role stops
//     issuing, drains copies and MMAs in flight, frees TMEM and reports
//     DIFFATTN_ERR_TIMEOUT.
#include "common.cuh"
#include "kernels.h"
#include "tma_host.cuh"

namespace diffattn {

namespace {
constexpr int BM = 128;                  // queries per CTA
constexpr int SUB = 64;                  // queries per sub-tile
constexpr int BN = 128;                  // keys per tile
constexpr int HALF = 128 * 128;          // one [128 rows x 64 bf16] swizzled block (16 KB)
constexpr int KSTAGES = 2, VSTAGES = 2;
constexpr int Q_OFF = 0;                 // sub-tile x at x * 2 * HALF
constexpr int K_OFF = Q_OFF + 4 * HALF;  // stage s: 2 blocks (d halves)
constexpr int V_OFF = K_OFF + KSTAGES * 2 * HALF;  // stage s: 2 blocks (value column halves)
constexpr int MISC_OFF = V_OFF + VSTAGES * 2 * HALF;
constexpr int MISC_BYTES = 1024;
constexpr int SMEM_BYTES = MISC_OFF + MISC_BYTES + 1024;
constexpr int NUM_THREADS = 384;
constexpr int REGS_SOFTMAX = 200, REGS_OTHER = 104;
constexpr int TMEM_COLS = 512;
constexpr float RESCALE_LOG2 = 8.0f;
// Of every 4 pairs of exponentials, POLY go to the FMA pipe (kernel template argument): 1
// for launches that run at full clock, 0 for launches long enough to run under the power
// cap, where the polynomial's extra instructions cost more energy than the MUFU work they
// save (measured: N = 65536 1.1% faster with 0, N = 16384 1.3% slower).
constexpr double kLongLaunchFlops = 2e13;
constexpr int QBAND = 32;              // query tiles per band of the CTA order

struct Misc {
  uint64_t q_full[2];
  uint64_t k_full[KSTAGES], k_empty[KSTAGES];
  uint64_t v_full[VSTAGES], v_empty[VSTAGES];
  uint64_t s_full[2];  // [sub-tile] scores of the current key tile are in TMEM
  uint64_t p_full[2];  // [sub-tile] P of the current key tile is in TMEM (128 arrivals)
  uint64_t o_full[2];  // [sub-tile] its last P.V MMA has completed
  uint32_t tmem_base;
  int abort;
  int seq_q0, seq_bc, seq_nq;  // the tile's sequence, for the epilogue's stores
};
static_assert(sizeof(Misc) <= MISC_BYTES, "misc region");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_OTHER == NUM_THREADS * 168, "register split");

constexpr unsigned FULL = 0xffffffffu;

// descriptor of the same operand layout `bytes` further on (start address field, bits 0-13;
// shared-memory addresses stay below 2^18, so the field never carries)
__device__ __forceinline__ uint64_t desc_at(uint64_t desc, uint32_t bytes) {
  return desc + (uint64_t)(bytes >> 4);
}
}  // namespace

// WINDOW: a causal sliding window (a.window > 0). Without one every row sees key 0, the
// first key of the first tile, so the row state is set after tile 0 and the masks have
// only an upper end; that case compiles without the lower-end and unset-row checks.
// VARLEN: a variable-length batch (a.cu_q != nullptr); the fixed-length instantiation
// takes its sizes from the parameters alone.
// STATS: the statistics pass of the backward (fixed length only): the epilogue writes the
// log-sum-exps and deltas described at PrefillArgs::st instead of the output.
// TRAIN: the training forward (fixed length only): the output, and for the backward the
// branch-2 output O_2 / l_2 (PrefillArgs::tr_o2) and both log-sum-exps (tr_lse).
template <bool WINDOW, bool VARLEN, bool STATS = false, bool TRAIN = false, int POLY = 1>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_v2_kernel(const __grid_constant__ TcMaps maps, const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + MISC_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile -> (q-tile, unit, batch). The query tiles go in bands of QBAND, the heaviest
  // causal band first; inside a band, KV group by KV group (batch entry, KV head), each
  // group's tiles heaviest first and the pairs of a tile together. So the CTAs in flight
  // read the keys and values of one or two KV heads, which stay in L2, and the tiles that
  // are handed out last are the lightest.
  const int n_qt = (a.N + BM - 1) / BM;
  const int ppg = a.group / 2;                    // pairs per KV head
  const int n_kvh = a.units / ppg;
  const int per_band = QBAND * ppg * n_kvh * a.B;
  const int band = (int)(blockIdx.x / per_band);
  const int r_b = (int)(blockIdx.x - (unsigned)band * per_band);
  const int band_len = min(QBAND, n_qt - QBAND * band);
  const int grp = r_b / (band_len * ppg), r_g = r_b - grp * (band_len * ppg);
  const int qt_i = QBAND * band + r_g / ppg;
  const int qt = a.causal ? n_qt - 1 - qt_i : qt_i;
  const int u = (grp % n_kvh) * ppg + r_g % ppg;
  const int b = grp / n_kvh;
  const int q0 = qt * BM;
  // the sequence of this tile (a variable-length batch packs several into one tensor);
  // the whole CTA leaves before any setup when the tile lies past its sequence
  const SeqRange sr = seq_range<VARLEN>(a, b);
  if (VARLEN && (!sr.ok || q0 >= sr.nq)) {
    if (!sr.ok && threadIdx.x == 0 && q0 == 0 && u == 0)
      report_status(a.dev_status, DIFFATTN_ERR_INVALID_ARG);
    return;
  }
  // query i sits at key position i + off (chunked prefill: the last nq of nk positions);
  // this tile sees keys klo .. khi, in key tiles j_lo .. j_lo + n_kt - 1
  const int off = sr.nk - sr.nq;
  const int khi = a.causal ? min(q0 + BM - 1 + off, sr.nk - 1) : sr.nk - 1;
  const int klo = WINDOW ? max(0, q0 + off - a.window + 1) : 0;
  const int j_lo = klo / BN;
  const int n_kt = (khi + BN) / BN - j_lo;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&ms.q_full[x], 1);
      mbar_init(&ms.s_full[x], 1);
      mbar_init(&ms.p_full[x], 128);
      mbar_init(&ms.o_full[x], 1);
    }
    for (int s = 0; s < KSTAGES; ++s) {
      mbar_init(&ms.k_full[s], 1);
      mbar_init(&ms.k_empty[s], 1);
    }
    for (int s = 0; s < VSTAGES; ++s) {
      mbar_init(&ms.v_full[s], 1);
      mbar_init(&ms.v_empty[s], 1);
    }
    ms.abort = 0;
    if (VARLEN) {
      ms.seq_q0 = sr.qrow0;
      ms.seq_bc = sr.bc;
      ms.seq_nq = sr.nq;
    }
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

  // query heads 2u, 2u+1 and their KV head
  const int kvh = (2 * u) / a.group;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
    if (warp == 8 && lane == 0) {
      // ------------------------------ TMA producer -----------------------------------
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      for (int x = 0; x < 2; ++x) {
        uint8_t* qd = smem + Q_OFF + x * 2 * HALF;
        const int t0 = q0 + x * SUB;
        // rows in TMEM-lane order: 16-row groups alternate branch 1 / branch 2
        mbar_arrive_expect_tx(&ms.q_full[x], 2 * HALF);
        for (int hf = 0; hf < 2; ++hf)
          for (int g = 0; g < 8; ++g)
            tma_load_4d(qd + hf * HALF + g * 2048, &maps.q, &ms.q_full[x], 64 * hf,
                        2 * u + (g & 1), sr.qrow0 + t0 + 16 * (g >> 1), sr.bc);
      }
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kt && !*abort_flag; ++j) {
        const int ks = j % KSTAGES;
        if (!mbar_wait(&ms.k_empty[ks], ((j / KSTAGES) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&ms.k_full[ks], 2 * HALF);
        uint8_t* kd = smem + K_OFF + ks * 2 * HALF;
        tma_load_4d(kd, &maps.k, &ms.k_full[ks], 0, kvh, sr.krow0 + (j_lo + j) * BN, sr.bc);
        tma_load_4d(kd + HALF, &maps.k, &ms.k_full[ks], 64, kvh, sr.krow0 + (j_lo + j) * BN, sr.bc);
        issued_k = j + 1;
        const int vs = j % VSTAGES;
        if (!mbar_wait(&ms.v_empty[vs], ((j / VSTAGES) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&ms.v_full[vs], 2 * HALF);
        uint8_t* vd = smem + V_OFF + vs * 2 * HALF;
        tma_load_4d(vd, &maps.v, &ms.v_full[vs], 0, kvh, sr.krow0 + (j_lo + j) * BN, sr.bc);
        tma_load_4d(vd + HALF, &maps.v, &ms.v_full[vs], 64, kvh, sr.krow0 + (j_lo + j) * BN, sr.bc);
        issued_v = j + 1;
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA's shared memory goes away
        mbar_wait_drain(&ms.q_full[0], 0);
        mbar_wait_drain(&ms.q_full[1], 0);
        for (int j = max(0, issued_k - KSTAGES); j < issued_k; ++j)
          mbar_wait_drain(&ms.k_full[j % KSTAGES], (j / KSTAGES) & 1);
        for (int j = max(0, issued_v - VSTAGES); j < issued_v; ++j)
          mbar_wait_drain(&ms.v_full[j % VSTAGES], (j / VSTAGES) & 1);
      }
    } else if (warp == 9 && lane == 0) {
      // ------------------------------ MMA issuer -------------------------------------
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, false, true);
      // K-major operands (Q, K): 8-row groups 1024 B apart, k-step = 32 B inside the swizzle
      // atom. V (B of P.V) is MN-major: 16 keys per k-step (2048 B), column blocks HALF apart.
      const uint64_t qdesc = sw128_desc(smem_u32(smem + Q_OFF), 16, 1024);
      const uint64_t kdesc = sw128_desc(smem_u32(smem + K_OFF), 16, 1024);
      const uint64_t vdesc = sw128_desc(smem_u32(smem + V_OFF), HALF, 1024);
      auto issue_s = [&](int x, int j) {
        const uint64_t kd = desc_at(kdesc, (j % KSTAGES) * 2 * HALF);
        const uint64_t qd = desc_at(qdesc, x * 2 * HALF);
        const uint32_t d = tmem + 256u * x;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          umma_ss(d, desc_at(qd, off), desc_at(kd, off), IDESC_S, kk > 0);
        }
        tc_commit(&ms.s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {
        const uint64_t vd = desc_at(vdesc, (j % VSTAGES) * 2 * HALF);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + 256u * x + 128u, tmem + 256u * x + kk * 8, desc_at(vd, kk * 2048),
                  IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool done0 = false, done1 = false;
      bool ok = mbar_wait(&ms.q_full[0], 0, abort_flag) && mbar_wait(&ms.k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        ok = mbar_wait(&ms.q_full[1], 0, abort_flag);
      }
      if (ok) {
        tc_fence_after();
        issue_s(1, 0);
        tc_commit(&ms.k_empty[0]);
      }
      for (int j = 0; j < n_kt && ok; ++j) {
        const int vs = j % VSTAGES;
        const int ks = (j + 1) % KSTAGES;
        if (!(ok = mbar_wait(&ms.v_full[vs], (j / VSTAGES) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&ms.p_full[0], j & 1, abort_flag))) break;
        tc_fence_after();
        issue_pv(0, j);
        if (j + 1 == n_kt) {
          tc_commit(&ms.o_full[0]);
          done0 = true;
        } else {
          if (!(ok = mbar_wait(&ms.k_full[ks], ((j + 1) / KSTAGES) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s(0, j + 1);  // S/P block 0 is rewritten after the P.V MMAs above read it
        }
        if (!(ok = mbar_wait(&ms.p_full[1], j & 1, abort_flag))) break;
        tc_fence_after();
        issue_pv(1, j);
        tc_commit(&ms.v_empty[vs]);
        if (j + 1 == n_kt) {
          tc_commit(&ms.o_full[1]);
          done1 = true;
        } else {
          issue_s(1, j + 1);
          tc_commit(&ms.k_empty[ks]);
        }
      }
      // on an abort, these still arrive once every MMA issued above has completed
      if (!done0) tc_commit(&ms.o_full[0]);
      if (!done1) tc_commit(&ms.o_full[1]);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // --------------------------- softmax warpgroups ------------------------------------
    // Thread (warp wq, lane) owns query tq = 16 wq + lane % 16 of its sub-tile and half hh =
    // lane / 16 of the key tile and of the value columns (64 each): it holds BOTH branches'
    // scores of those keys (the split 16-lane TMEM loads read the branch-1 row, lanes 32 wq
    // + lane % 16, and the branch-2 row, 16 lanes further on), so p1 - c p2 is formed in
    // registers. The two halves of a query exchange only their maxima and sums (lane ^ 16).
    const int x = warp >> 2;                       // sub-tile
    const int wq = warp & 3;                       // 32-lane group of TMEM
    const int hh = (lane >> 4) & 1;                // half: keys / value columns 64 hh .. 64 hh + 63
    const int tq = wq * 16 + (lane & 15);          // query within the sub-tile
    const int qi = q0 + x * SUB + tq;
    const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t s1_addr = lane_addr + 256u * x;  // branch-1 rows: S, then P over 64 columns
    const uint32_t s2_addr = s1_addr + (16u << 16); // branch-2 rows
    const uint32_t o1_addr = s1_addr + 128u;        // D (branch-1 rows)
    const uint32_t o2_addr = s2_addr + 128u;        // O_2 (branch-2 rows)
    const float sl2 = 1.4426950408889634f * rsqrtf((float)a.d);  // log2(e)/sqrt(d)
    const float lam = a.lambda[u];
    // visible keys of this query: vlo .. vis (causal: up to its own position, clamped for
    // the padding rows of the last tile; window: the last `window` of those)
    const int vis = a.causal ? min(qi + off, sr.nk - 1) : sr.nk - 1;
    const int vlo = WINDOW ? max(0, vis - a.window + 1) : 0;
    float m1 = -INFINITY, m2 = -INFINITY, l1 = 0.f, l2 = 0.f;  // identical in both halves
    float c = 0.f;
    bool ok = true;

    for (int j = 0; j < n_kt; ++j) {
      if (ok) ok = mbar_wait(&ms.s_full[x], j & 1, abort_flag);
      if (!(ok = __all_sync(FULL, ok))) break;
      tc_fence_after();
      float p[2 * SUB];  // p[e]: branch 1, key 64 hh + e; p[64 + e]: branch 2, same key
      tmem_ld16x2_32f_split<64>(s1_addr, p);
      tmem_ld16x2_32f_split<64>(s1_addr + 32, p + 32);
      tmem_ld16x2_32f_split<64>(s2_addr, p + 64);
      tmem_ld16x2_32f_split<64>(s2_addr + 32, p + 96);
      tmem_wait_ld();
      const int lim = vis - (j_lo + j) * BN - 64 * hh, llim = vlo - (j_lo + j) * BN - 64 * hh;
      if (lim < 63 || (WINDOW && llim > 0)) {
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e > lim || (WINDOW && e < llim)) p[e] = p[64 + e] = -INFINITY;
      }
      float u0 = -INFINITY, u1 = -INFINITY, w0 = -INFINITY, w1 = -INFINITY;
#pragma unroll
      for (int e = 0; e < 64; e += 4) {
        u0 = fmax3(u0, p[e + 0], p[e + 1]);
        u1 = fmax3(u1, p[e + 2], p[e + 3]);
        w0 = fmax3(w0, p[64 + e + 0], p[64 + e + 1]);
        w1 = fmax3(w1, p[64 + e + 2], p[64 + e + 3]);
      }
      float t1 = fmaxf(u0, u1), t2 = fmaxf(w0, w1);
      t1 = fmaxf(t1, __shfl_xor_sync(FULL, t1, 16)) * sl2;
      t2 = fmaxf(t2, __shfl_xor_sync(FULL, t2, 16)) * sl2;
      // lazy maxima: raised only on growth by more than 2^8 (or when unset)
      const bool had = WINDOW ? m1 != -INFINITY : j > 0;  // the query saw a visible key before
      const bool r1 = (t1 > m1 + RESCALE_LOG2) || !had, r2 = (t2 > m2 + RESCALE_LOG2) || !had;
      const float n1 = r1 ? fmaxf(t1, m1) : m1, n2 = r2 ? fmaxf(t2, m2) : m2;
      const float a1 = (r1 && had) ? ex2(m1 - n1) : 1.f, a2 = (r2 && had) ? ex2(m2 - n2) : 1.f;
      m1 = n1;
      m2 = n2;
      // p = 2^(s sl2 - m), in place (0 for every key while the query has none visible); in
      // every group of 8 keys the last POLY pairs go to the FMA pipe, the rest to MUFU
      const float nm1 = (WINDOW && m1 == -INFINITY) ? 0.f : -m1;
      const float nm2 = (WINDOW && m2 == -INFINITY) ? 0.f : -m2;
      float sa = 0.f, sb = 0.f, sc = 0.f, sd = 0.f;
#pragma unroll
      for (int e = 0; e < 64; e += 8) {
#pragma unroll
        for (int br = 0; br < 2; ++br) {
          float* pb = p + 64 * br + e;
          const float nm = br ? nm2 : nm1;
          float xv[8];
#pragma unroll
          for (int i = 0; i < 8; i += 2) ffma2(xv[i], xv[i + 1], pb[i], pb[i + 1], sl2, sl2, nm, nm);
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            if (i >= 8 - 2 * POLY) {
              exp2_fma2(pb[i], pb[i + 1], xv[i], xv[i + 1]);
            } else {
              pb[i] = ex2(xv[i]);
              pb[i + 1] = ex2(xv[i + 1]);
            }
          }
          if (br == 0) {
            fadd2(sa, sb, sa, sb, pb[0], pb[1]);
            fadd2(sa, sb, sa, sb, pb[2], pb[3]);
            fadd2(sa, sb, sa, sb, pb[4], pb[5]);
            fadd2(sa, sb, sa, sb, pb[6], pb[7]);
          } else {
            fadd2(sc, sd, sc, sd, pb[0], pb[1]);
            fadd2(sc, sd, sc, sd, pb[2], pb[3]);
            fadd2(sc, sd, sc, sd, pb[4], pb[5]);
            fadd2(sc, sd, sc, sd, pb[6], pb[7]);
          }
        }
      }
      // tile sums over both halves: a + b is the same float in either order, so both halves
      // of the query keep bit-identical l_1, l_2 (and so take the same decisions below)
      const float s1h = sa + sb, s2h = sc + sd;
      l1 = l1 * a1 + (s1h + __shfl_xor_sync(FULL, s1h, 16));
      l2 = l2 * a2 + (s2h + __shfl_xor_sync(FULL, s2h, 16));

      // target c = lambda l_1 / l_2 (sums including this tile); under max updates c follows
      // c a_1 / a_2, which leaves D unchanged; reset to the target when it leaves
      // [0.8, 1.25] times it (the query's first tile with a visible key always takes the
      // target: D and O_2 are still 0).
      const float cst = (WINDOW && !(l2 > 0.f)) ? lam : lam * __fdiv_rn(l1, l2);  // exact ratio: identical branches give c = lambda
      float cn = cst, kc = 0.f;
      bool need = false;
      if (had) {
        const float cev = (a1 == a2) ? c : c * __fdividef(a1, a2);
        const float ra = fabsf(cev), rt = fabsf(cst);
        const bool reset = !(ra >= 0.8f * rt && ra <= 1.25f * rt);
        cn = reset ? cst : cev;
        if (reset) kc = __fsub_rn(__fmul_rn(a1, c), __fmul_rn(a2, cn));
        need = (a1 != 1.f) || (a2 != 1.f) || (kc != 0.f);
      }
      c = cn;
      // P rows (bf16 pairs over the first 64 columns of the S block): branch 1 p1 - c p2,
      // branch 2 p2; this half's 64 keys are columns 32 hh .. 32 hh + 31. Every column
      // written here was read by this warp's loads above, which have completed.
      {
        const float nc = -c;
        uint32_t pk1[32], pk2[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          float v0, v1;
          ffma2(v0, v1, p[64 + e], p[64 + e + 1], nc, nc, p[e], p[e + 1]);
          pk1[e / 2] = pack_bf16(v0, v1);
          pk2[e / 2] = pack_bf16(p[64 + e], p[64 + e + 1]);
        }
        tmem_st16x2_32_split<32>(s1_addr, pk1);
        tmem_st16x2_32_split<32>(s2_addr, pk2);
      }
      if (WINDOW || j > 0) {
        // the whole warp rescales (a query with nothing to do has a_1 = a_2 = 1, kc = 0):
        // D <- a_1 D + kc O_2, O_2 <- a_2 O_2 over this half's 64 value columns. The score
        // MMA that filled S was issued after this sub-tile's previous P.V MMAs, so its
        // completion implies theirs; the next P.V MMA waits for p_full below.
        if (__any_sync(FULL, need)) {
#pragma unroll 1
          for (int ch = 0; ch < 2; ++ch) {
            float dv[32], ov[32];
            tmem_ld16x2_32f_split<64>(o1_addr + ch * 32, dv);
            tmem_ld16x2_32f_split<64>(o2_addr + ch * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              dv[e] = fmaf(kc, ov[e], a1 * dv[e]);
              ov[e] *= a2;
            }
            tmem_st16x2_32f_split<64>(o1_addr + ch * 32, dv);
            tmem_st16x2_32f_split<64>(o2_addr + ch * 32, ov);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ms.p_full[x]);
    }

    // ------------------------------- epilogue ----------------------------------------
    if (ok) ok = mbar_wait(&ms.o_full[x], 0, abort_flag);
    ok = __all_sync(FULL, ok);
    const float inv1 = 1.f / l1, inv2 = 1.f / l2;
    // o = D / l_1 + O_2 (c / l_1 - lambda / l_2); products rounded on their own so that
    // identical branches with lambda = 1 give exactly 0
    const float coef = __fsub_rn(__fmul_rn(c, inv1), __fmul_rn(lam, inv2));
    // this thread writes value columns 64 hh .. 64 hh + 63 of its query
    float y[64];  // the output, or (STATS) the incoming gradient dy of the same columns
    float e1 = 0.f, e2 = 0.f;
    if constexpr (STATS) {
      const int64_t dy_off = (int64_t)b * a.st_dys[0] + (int64_t)qi * a.st_dys[1] +
                             (int64_t)u * a.st_dys[2] + hh * 64;
      if (ok && qi < a.N && in_bounds(dy_off, 64, a.ext_st_dy, a.dev_status, a.dbg_status)) {
        const uint4* g4 = reinterpret_cast<const uint4*>(
            static_cast<const __nv_bfloat16*>(a.st_dy) + dy_off);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 w = g4[v];
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            y[v * 8 + 2 * e] = __uint_as_float(wv[e] << 16);
            y[v * 8 + 2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) y[e] = 0.f;
      }
    }
    if (ok) {
      tc_fence_after();
      const float c1 = c * inv1;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float dv[32], ov[32];
        tmem_ld16x2_32f_split<64>(o1_addr + ch * 32, dv);
        tmem_ld16x2_32f_split<64>(o2_addr + ch * 32, ov);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if constexpr (STATS) {
            // O_1 / l_1 = (D + c O_2) / l_1 and O_2 / l_2 at this column, against dy
            e1 = fmaf(y[ch * 32 + e], __fmaf_rn(ov[e], c1, dv[e] * inv1), e1);
            e2 = fmaf(y[ch * 32 + e], ov[e] * inv2, e2);
          } else {
            y[ch * 32 + e] = __fmaf_rn(ov[e], coef, __fmul_rn(dv[e], inv1));
          }
        }
        if constexpr (TRAIN) {
          // O_2 / l_2 of these 32 columns, in out's layout
          const int64_t o2_off = (int64_t)b * a.os[0] + (int64_t)qi * a.os[1] + (int64_t)u * a.os[2] +
                                 hh * 64 + ch * 32;
          if (qi < a.N && in_bounds(o2_off, 32, a.ext_out, a.dev_status, a.dbg_status)) {
            uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.tr_o2) + o2_off);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_bf16(ov[v * 8 + 0] * inv2, ov[v * 8 + 1] * inv2);
              w.y = pack_bf16(ov[v * 8 + 2] * inv2, ov[v * 8 + 3] * inv2);
              w.z = pack_bf16(ov[v * 8 + 4] * inv2, ov[v * 8 + 5] * inv2);
              w.w = pack_bf16(ov[v * 8 + 6] * inv2, ov[v * 8 + 7] * inv2);
              o4[v] = w;
            }
          }
        }
      }
    }
    if constexpr (TRAIN) {
      const int64_t rl = (((int64_t)b * a.units + u) * a.N + qi) * 2;
      if (ok && hh == 0 && qi < a.N && in_bounds(rl, 2, a.ext_tr_lse, a.dev_status, a.dbg_status))
        *reinterpret_cast<float2*>(a.tr_lse + rl) = make_float2(m1 + log2f(l1), m2 + log2f(l2));
    }
    if constexpr (STATS) {
      // the query's two halves add their column ranges; lse_b = m_b + log2 l_b (log2 domain)
      e1 += __shfl_xor_sync(FULL, e1, 16);
      e2 += __shfl_xor_sync(FULL, e2, 16);
      if (ok && hh == 0 && qi < a.N) {
        const int64_t r = ((int64_t)b * a.units + u) * a.st_rows + qi;
        const int64_t rl = ((int64_t)b * a.units + u) * a.N + qi;
        if (in_bounds(r * 4, 4, a.ext_st, a.dev_status, a.dbg_status))
          *reinterpret_cast<float4*>(a.st + r * 4) =
              make_float4(m1 + log2f(l1), m2 + log2f(l2), e1, e2);
        if (in_bounds(rl, 1, a.ext_st_dl, a.dev_status, a.dbg_status)) a.st_dl[rl] = -e2;
      }
    }
    // (a variable-length tile reads its sequence back from shared memory, keeping the
    // registers of the key loop free)
    const int o_nq = VARLEN ? ms.seq_nq : a.N, o_b = VARLEN ? ms.seq_bc : b;
    const int o_q0 = VARLEN ? ms.seq_q0 : 0;
    const int64_t o_off = (int64_t)o_b * a.os[0] + (int64_t)(o_q0 + qi) * a.os[1] +
                          (int64_t)u * a.os[2] + hh * 64;
    if (!STATS && ok && qi < o_nq && in_bounds(o_off, 64, a.ext_out, a.dev_status, a.dbg_status)) {
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.out) + o_off;
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    if (*abort_flag) {
      mbar_wait_drain(&ms.o_full[0], 0);
      mbar_wait_drain(&ms.o_full[1], 0);
      if (lane == 0) report_status(a.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_prefill_v2(const PrefillArgs& a, cudaStream_t stream) {
  if (a.variant != DIFFATTN_V2 || a.d != 128 || a.group % 2 != 0) return cudaErrorNotSupported;
  TcMaps maps;
  // q [B, N, Hq, 128], k, v [B, N, Hkv, 128]; Q boxes of 16 queries of one head (the
  // TMEM-lane row order), K and V boxes of 128 keys
  // a variable-length batch is one packed sequence of rows to the tensor maps
  const int rq = a.cu_q ? a.total_q : a.N, rk = a.cu_q ? a.total_k : a.Nk, nb = a.cu_q ? 1 : a.B;
  if (!make_map(&maps.q, a.q, 128, a.Hq, rq, nb, a.qs, 16)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, 128, a.Hkv, rk, nb, a.ks, BN)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, 128, a.Hkv, rk, nb, a.vs, BN)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const void* fns[5] = {(const void*)prefill_v2_kernel<false, false>, (const void*)prefill_v2_kernel<true, false>,
                          (const void*)prefill_v2_kernel<false, true>, (const void*)prefill_v2_kernel<true, true>,
                          (const void*)prefill_v2_kernel<false, false, false, false, 0>};
    for (const void* fn : fns) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    if (dev < 64) attr_set[dev] = true;
  }
  const long long tiles = (long long)((a.N + BM - 1) / BM) * a.units * a.B;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const bool window = a.causal && a.window > 0, varlen = a.cu_q != nullptr;
  const dim3 grid((unsigned)tiles);
  if (varlen) {
    if (window) prefill_v2_kernel<true, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
    else prefill_v2_kernel<false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  } else if (window) {
    prefill_v2_kernel<true, false><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  } else {
    // algorithmic FLOPs of the launch: 4 d per attended (query, key) pair and query head
    const double nq = a.N, nk = a.Nk;
    const double pairs = a.causal ? nq * (nk - nq) + nq * (nq + 1) / 2 : nq * nk;
    const double flops = 4.0 * a.d * a.Hq * (double)a.B * pairs;
    if (flops >= kLongLaunchFlops)
      prefill_v2_kernel<false, false, false, false, 0><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
    else
      prefill_v2_kernel<false, false><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  }
  return cudaGetLastError();
}

// The training forward over the same tiles (fixed-length batches): out, tr_o2 and tr_lse
// must be set.
cudaError_t launch_prefill_v2_train(const PrefillArgs& a, cudaStream_t stream) {
  if (a.variant != DIFFATTN_V2 || a.d != 128 || a.group % 2 != 0 || a.cu_q) return cudaErrorNotSupported;
  if (!a.out || !a.tr_o2 || !a.tr_lse) return cudaErrorInvalidValue;
  TcMaps maps;
  if (!make_map(&maps.q, a.q, 128, a.Hq, a.N, a.B, a.qs, 16)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, 128, a.Hkv, a.Nk, a.B, a.ks, BN)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, 128, a.Hkv, a.Nk, a.B, a.vs, BN)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const void* fns[2] = {(const void*)prefill_v2_kernel<false, false, false, true>,
                          (const void*)prefill_v2_kernel<true, false, false, true>};
    for (const void* fn : fns) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    if (dev < 64) attr_set[dev] = true;
  }
  const long long tiles = (long long)((a.N + BM - 1) / BM) * a.units * a.B;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const dim3 grid((unsigned)tiles);
  if (a.causal && a.window > 0)
    prefill_v2_kernel<true, false, false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  else
    prefill_v2_kernel<false, false, false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  return cudaGetLastError();
}

// The backward's statistics pass over the same tiles (fixed-length batches): st, st_dl and
// st_dy must be set; out is not written.
cudaError_t launch_prefill_v2_stats(const PrefillArgs& a, cudaStream_t stream) {
  if (a.variant != DIFFATTN_V2 || a.d != 128 || a.group % 2 != 0 || a.cu_q) return cudaErrorNotSupported;
  if (!a.st || !a.st_dl || !a.st_dy) return cudaErrorInvalidValue;
  TcMaps maps;
  if (!make_map(&maps.q, a.q, 128, a.Hq, a.N, a.B, a.qs, 16)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, 128, a.Hkv, a.Nk, a.B, a.ks, BN)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, 128, a.Hkv, a.Nk, a.B, a.vs, BN)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const void* fns[2] = {(const void*)prefill_v2_kernel<false, false, true>,
                          (const void*)prefill_v2_kernel<true, false, true>};
    for (const void* fn : fns) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    if (dev < 64) attr_set[dev] = true;
  }
  const long long tiles = (long long)((a.N + BM - 1) / BM) * a.units * a.B;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const dim3 grid((unsigned)tiles);
  if (a.causal && a.window > 0)
    prefill_v2_kernel<true, false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  else
    prefill_v2_kernel<false, false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace diffattn
