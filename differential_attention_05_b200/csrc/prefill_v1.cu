// prefill_v1.cu -- single-pass fused differential attention prefill on the sm_100a tensor
// cores, V1 (branch width d = 64, value width 2d = 128). V2 runs on the kernel in
// prefill_v2.cu.
//
// What it computes, per head and query row i:
//   A_b = softmax(Q_b K_b^T / sqrt(d)) over keys j <= i (causal) or all keys,  b = 1, 2
//   o   = (A_1 - lambda A_2) V,   then   o <- o / sqrt(mean(o^2) + eps) * (1 - lambda_init)
// ("Differential Attention (V2)", The Concept, "The difference idea" and "V1 vs V2";
//  "Attention Variants", Build It, Steps 1 and 4; Hugging Face post, "How?").
//
// Rounding the two branches' probabilities to bf16 separately and subtracting afterwards
// loses the difference when the branches nearly cancel (lambda near 1, similar maps): the
// 2^-9 rounding error of each map is amplified by about 1/(1 - lambda), and the per-head
// RMSNorm amplifies it again. So the kernel accumulates, per row,
//   D   = sum_j (p1_j - c p2_j) v_j      with c near lambda l_1 / l_2
//   O_2 = sum_j p2_j v_j
// where p_b = 2^(s_b log2(e)/sqrt(d) - m_b) and m_b is branch b's running maximum. The
// operand p1 - c p2 is formed in fp32 from the exact p1, p2 and rounded once, so it carries
// an error relative to the (small) difference itself. At the end
//   o = O_1/l_1 - lambda O_2/l_2 = D/l_1 + O_2 (c/l_1 - lambda/l_2),
// and the rounding error of O_2 enters only through c/l_1 - lambda/l_2, which vanishes as
// c is set to lambda l_1 / l_2 from the running sums (including the current key tile).
// D = O_1 - c O_2 is kept exact across updates: raising m_1 (factor a_1) or m_2 (factor a_2)
// and moving c to c' maps D -> a_1 D + (a_1 c - a_2 c') O_2 and O_2 -> a_2 O_2, done lazily
// -- a maximum is raised only when it grows by more than 2^8, and c is reset only when it
// leaves [0.8, 1.25] times its target.
//
// Layout of the work (one CTA per 128-query tile of one head, heaviest causal tiles first):
//   * keys in tiles of 64; S_1 = Q_1 K_1^T and S_2 = Q_2 K_2^T of a tile share one TMEM
//     buffer (2 x 64 columns), double-buffered, so the tensor core computes tile j+1 while
//     tile j is in the softmax; D and O_2 take the other 256 TMEM columns. (Stacking both
//     branches of 64 queries into one 128-row MMA, as the V2 kernel does, gains nothing
//     here: with K_1 != K_2 the score MMAs would be two M = 64 instructions, which cost
//     what the M = 128, N = 64 ones do.)
//   * warps 4-7 own branch 2: for every key tile they form p2 over the tile's 64 keys,
//     write it in fp32 over their own score columns and post (max, rescale factor, sum) of
//     each row through shared memory and an mbarrier, then move on to the next tile.
//     Warps 0-3 own branch 1: they form p1, take branch 2's tile, choose c, keep D exact
//     (rescales), and write both bf16 operands over S_1; the P.V MMAs read them straight
//     from TMEM. Thread t owns TMEM lane t = query row t, so row max and row sum need no
//     shuffles, and branch 2 running a tile ahead keeps both warpgroups busy.
//   * warp 8: TMA loads (128-byte swizzle, no multicast) of Q once and K, V in 4-stage
//     rings; each V tile feeds both P.V products.
//   * only the branch-1 warpgroup and the MMA warp rescale / read the accumulators.
//   * warp 9: TMEM allocation and every tcgen05.mma / commit.
//   * registers are re-split after launch (setmaxnreg): 208 for the softmax warpgroups,
//     88 for the third; 2 * 208 + 88 = 3 * 168, the launch allocation.
//   * every mbarrier wait is bounded; a timeout raises an abort flag so every role stops
//     issuing (the softmax warpgroups pass the same number of named barriers), drains
//     copies and MMAs in flight, frees TMEM and reports DIFFATTN_ERR_TIMEOUT.
#include "common.cuh"
#include "kernels.h"
#include "tma_host.cuh"

namespace diffattn {

namespace {
constexpr int BM = 128;                  // queries per tile
constexpr int BN = 64;                   // keys per tile
constexpr int QBLK = 128 * 128;          // [128 rows x 64 bf16], 128-byte swizzle
constexpr int KBLK = 64 * 128;           // [64 rows x 64 bf16]
constexpr int STAGES = 4;
constexpr int Q_OFF = 0;                 // Q_1 blocks at 0 (,16K); Q_2 at 32K (,48K)
constexpr int K_OFF = 4 * QBLK;
constexpr int V_OFF = K_OFF + STAGES * 2 * KBLK;
constexpr int MISC_OFF = V_OFF + STAGES * 2 * KBLK;
constexpr int MISC_BYTES = 12288;
constexpr int SMEM_BYTES = MISC_OFF + MISC_BYTES + 1024;
constexpr int NUM_THREADS = 384;
constexpr int REGS_SOFTMAX = 208, REGS_OTHER = 88;
constexpr int POLY_PAIRS = 0;  // of every 4 pairs of exponentials, on the FMA pipe
constexpr int TMEM_COLS = 512;
constexpr uint32_t COL_D = 256, COL_O2 = 384;
constexpr float RESCALE_LOG2 = 8.0f;

struct Misc {
  uint64_t q_full;
  uint64_t k_full[STAGES], k_empty[STAGES];
  uint64_t v_full[STAGES], v_empty[STAGES];
  uint64_t s_full[2];
  // one per S buffer: a buffer is reused two tiles later only after these were consumed,
  // so a waiter can never see two completed phases of the same barrier
  uint64_t p2_ready[2];  // branch 2 posted p2 (TMEM) and its row state (below) for a tile
  uint64_t p_full[2];    // the P.V operands of a tile are in TMEM
  uint64_t pv_done;  // the P.V MMAs of a tile have completed
  uint64_t o_full;   // every MMA has completed
  uint32_t tmem_base;
  int abort;
  int seq_q0, seq_bc, seq_nq;  // the tile's sequence, for the epilogue's stores
  float h_a2[2][BM];      // [tile parity][row] branch 2: rescale factor of the tile
  float h_l2[2][BM];      //                    running sum including the tile
  float ex_l[2][BM];      // epilogue: [branch][row] row sums
  float ex_c[BM];         // epilogue: c
  float ssx[2][BM];       // V1 norm: partial sums of squares
  float ex_m[2][BM];      // statistics pass: [branch][row] maxima
  float ex_s[4][2][BM];   //                  [quantity][half][row] partial dot products
};
static_assert(sizeof(Misc) <= MISC_BYTES, "misc region");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
}  // namespace

__device__ __forceinline__ void bar_softmax() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// WINDOW: a causal sliding window (a.window > 0). Without one every row sees key 0, the
// first key of the first tile, so the row state is set after tile 0 and the masks have
// only an upper end; that case compiles without the lower-end and unset-row checks.
// VARLEN: a variable-length batch (a.cu_q != nullptr); the fixed-length instantiation
// takes its sizes from the parameters alone.
// STATS: the statistics pass of the backward (fixed length only). Instead of the output the
// epilogue writes the gradient reaching o through the norm (PrefillArgs::st_do, bf16), the
// log-sum-exps, the deltas and the dlambda share (PrefillArgs::st, st_dl). The backward
// amplifies errors of o (the norm's backward projects dy against o, and on the usual inputs
// O_1 and O_2 are nearly parallel, so dlambda = -sum dO . O_2 keeps only their small
// difference), so here each P.V operand is split into a bf16 head and a bf16 remainder,
// x = hi(x) + lo(x) with |x - hi - lo| <= 2^-18 |x|, and both parts go through the MMA: D
// and O_2 come out as accurate as fp32 accumulation of fp32 probabilities.
template <bool WINDOW, bool VARLEN, bool STATS = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_v1_kernel(const __grid_constant__ TcMaps maps, const PrefillArgs a) {
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
    mbar_init(&ms.q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ms.k_full[s], 1); mbar_init(&ms.k_empty[s], 1);
      mbar_init(&ms.v_full[s], 1); mbar_init(&ms.v_empty[s], 1);
    }
    mbar_init(&ms.s_full[0], 1);
    mbar_init(&ms.s_full[1], 1);
    for (int f = 0; f < 2; ++f) {
      mbar_init(&ms.p2_ready[f], BM);
      mbar_init(&ms.p_full[f], BM);
    }
    mbar_init(&ms.pv_done, 1);
    mbar_init(&ms.o_full, 1);
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

  // TMA coordinates: head u, branch 1 / 2 at columns 0 / 64 of the [2d] rows of q and k

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
    if (warp == 8 && lane == 0) {
      // ------------------------------ TMA producer -----------------------------------
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      mbar_arrive_expect_tx(&ms.q_full, 2 * QBLK);
      tma_load_4d(smem + Q_OFF + 0 * QBLK, &maps.q, &ms.q_full, 0, u, sr.qrow0 + q0, sr.bc);   // q_1
      tma_load_4d(smem + Q_OFF + 2 * QBLK, &maps.q, &ms.q_full, 64, u, sr.qrow0 + q0, sr.bc);  // q_2
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kt && !*abort_flag; ++j) {
        const int st = j % STAGES;
        const uint32_t par = ((j / STAGES) & 1) ^ 1;
        if (!mbar_wait(&ms.k_empty[st], par, abort_flag)) break;
        mbar_arrive_expect_tx(&ms.k_full[st], 2 * KBLK);
        uint8_t* kd = smem + K_OFF + st * 2 * KBLK;  // k_1 | k_2
        tma_load_4d(kd, &maps.k, &ms.k_full[st], 0, u, sr.krow0 + (j_lo + j) * BN, sr.bc);
        tma_load_4d(kd + KBLK, &maps.k, &ms.k_full[st], 64, u, sr.krow0 + (j_lo + j) * BN, sr.bc);
        issued_k = j + 1;
        if (!mbar_wait(&ms.v_empty[st], par, abort_flag)) break;
        mbar_arrive_expect_tx(&ms.v_full[st], 2 * KBLK);
        uint8_t* vd = smem + V_OFF + st * 2 * KBLK;
        tma_load_4d(vd, &maps.v, &ms.v_full[st], 0, u, sr.krow0 + (j_lo + j) * BN, sr.bc);
        tma_load_4d(vd + KBLK, &maps.v, &ms.v_full[st], 64, u, sr.krow0 + (j_lo + j) * BN, sr.bc);
        issued_v = j + 1;
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA's shared memory goes away
        mbar_wait_drain(&ms.q_full, 0);
        for (int j = max(0, issued_k - STAGES); j < issued_k; ++j)
          mbar_wait_drain(&ms.k_full[j % STAGES], (j / STAGES) & 1);
        for (int j = max(0, issued_v - STAGES); j < issued_v; ++j)
          mbar_wait_drain(&ms.v_full[j % STAGES], (j / STAGES) & 1);
      }
    } else if (warp == 9 && lane == 0) {
      // ------------------------------ MMA issuer -------------------------------------
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, 128, false, true);
      const uint32_t qbase = smem_u32(smem + Q_OFF);
      const uint32_t kbase = smem_u32(smem + K_OFF);
      const uint32_t vbase = smem_u32(smem + V_OFF);
      // S_1, S_2 of key tile j into buffer f (columns 128 f, 128 f + 64)
      auto issue_s = [&](int f, int j) {
        const uint32_t kst = kbase + (j % STAGES) * 2 * KBLK;
#pragma unroll
        for (int br = 0; br < 2; ++br) {
          const uint32_t d = tmem + 128u * f + 64u * br;
          const uint32_t qb = qbase + br * 2 * QBLK;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(d, sw128_desc(qb + kk * 32, 16, 1024),
                    sw128_desc(kst + br * KBLK + kk * 32, 16, 1024), IDESC_S, kk > 0);
        }
        tc_commit(&ms.s_full[f]);
      };
      bool ok = mbar_wait(&ms.q_full, 0, abort_flag);
      for (int j = 0; j < 2 && j < n_kt && ok; ++j) {
        if (!(ok = mbar_wait(&ms.k_full[j], 0, abort_flag))) break;
        tc_fence_after();
        issue_s(j, j);
        tc_commit(&ms.k_empty[j]);
      }
      for (int j = 0; j < n_kt && ok; ++j) {
        const int f = j & 1, st = j % STAGES;
        if (!(ok = mbar_wait(&ms.v_full[st], (j / STAGES) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&ms.p_full[f], (j >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t vst = vbase + st * 2 * KBLK;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // B = V: MN-major, 16 keys per k-step (2048 B), column blocks 8 KB apart
          const uint64_t vd = sw128_desc(vst + kk * 2048, KBLK, 1024);
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          umma_ts(tmem + COL_D, tmem + 128u * f + kk * 8, vd, IDESC_PV, acc);
          umma_ts(tmem + COL_O2, tmem + 128u * f + 32u + kk * 8, vd, IDESC_PV, acc);
          if constexpr (STATS) {
            // the remainders, over S_2's columns: keys 32 h .. 32 h + 31 at 64 + 32 h (x)
            // and 64 + 32 h + 16 (p2)
            const uint32_t lo = 128u * f + 64u + 32u * (kk >> 1) + 8u * (kk & 1);
            umma_ts(tmem + COL_D, tmem + lo, vd, IDESC_PV, 1u);
            umma_ts(tmem + COL_O2, tmem + lo + 16u, vd, IDESC_PV, 1u);
          }
        }
        tc_commit(&ms.pv_done);
        tc_commit(&ms.v_empty[st]);
        if (j + 2 < n_kt) {
          const int s2 = (j + 2) % STAGES;
          if (!(ok = mbar_wait(&ms.k_full[s2], ((j + 2) / STAGES) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s(f, j + 2);  // buffer f is free once the P.V MMAs above have read it
          tc_commit(&ms.k_empty[s2]);
        }
      }
      tc_commit(&ms.o_full);  // arrives once every MMA issued above has completed
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // --------------------------- softmax warpgroups ------------------------------------
    const int wg = warp >> 2;                 // 0: branch 1 (+ operands), 1: branch 2
    const int row = (warp & 3) * 32 + lane;   // TMEM lane == query row
    const int qi = q0 + row;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = 1.4426950408889634f * rsqrtf((float)a.d);  // log2(e)/sqrt(d)
    const float lam = a.lambda[u];
    // visible keys of this row: vlo .. vis (causal: up to its own position; window: the
    // last `window` of those)
    const int vis = a.causal ? min(qi + off, sr.nk - 1) : sr.nk - 1;
    const int vlo = WINDOW ? max(0, vis - a.window + 1) : 0;
    // the same bounds relative to the first key of this tile's range
    const int vis0 = vis - j_lo * BN, vlo0 = vlo - j_lo * BN;
    float m = -INFINITY, l = 0.f;             // this warpgroup's branch
    float c = 0.f;                            // branch 1 warpgroup only
    bool ok = true;

    for (int j = 0; j < n_kt; ++j) {
      const int f = j & 1;
      const uint32_t sb = lane_addr + 128u * f;  // S_1 at +0, S_2 at +64
      if (ok) ok = mbar_wait(&ms.s_full[f], (j >> 1) & 1, abort_flag);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      // this branch's 64 scores of the tile
      float p[BN];
      tmem_ld32f(sb + 64u * wg, p);
      tmem_ld32f(sb + 64u * wg + 32, p + 32);
      tmem_wait_ld();
      const int lim = vis0 - j * BN, llim = vlo0 - j * BN;
      if (lim < BN - 1 || (WINDOW && llim > 0)) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e > lim || (WINDOW && e < llim)) p[e] = -INFINITY;
      }
      float c0 = -INFINITY, c1 = -INFINITY, c2 = -INFINITY, c3 = -INFINITY;
#pragma unroll
      for (int e = 0; e < BN; e += 8) {
        c0 = fmax3(c0, p[e + 0], p[e + 1]);
        c1 = fmax3(c1, p[e + 2], p[e + 3]);
        c2 = fmax3(c2, p[e + 4], p[e + 5]);
        c3 = fmax3(c3, p[e + 6], p[e + 7]);
      }
      const float t = fmax3(fmaxf(c0, c1), c2, c3) * sl2;
      // lazy maximum: raised only on growth by more than 2^8 (or when unset)
      const bool had = WINDOW ? m != -INFINITY : j > 0;  // the row saw a visible key before
      const bool r = (t > m + RESCALE_LOG2) || !had;
      const float n = r ? fmaxf(t, m) : m;
      const float al = (r && had) ? ex2(m - n) : 1.f;
      m = n;
      // p = 2^(s sl2 - m), in place (0 for every key while the row has none visible); in
      // every group of 8 keys the last POLY_PAIRS pairs go to the FMA pipe, the rest to MUFU
      float sa = 0.f, sb2 = 0.f, sc2 = 0.f, sd = 0.f;
      const float nm = (WINDOW && m == -INFINITY) ? 0.f : -m;
#pragma unroll
      for (int e = 0; e < BN; e += 8) {
        float xv[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) ffma2(xv[i], xv[i + 1], p[e + i], p[e + i + 1], sl2, sl2, nm, nm);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          if (i >= 8 - 2 * POLY_PAIRS) {
            exp2_fma2(p[e + i], p[e + i + 1], xv[i], xv[i + 1]);
          } else {
            p[e + i] = ex2(xv[i]);
            p[e + i + 1] = ex2(xv[i + 1]);
          }
        }
        fadd2(sa, sb2, sa, sb2, p[e], p[e + 1]);
        fadd2(sc2, sd, sc2, sd, p[e + 2], p[e + 3]);
        fadd2(sa, sb2, sa, sb2, p[e + 4], p[e + 5]);
        fadd2(sc2, sd, sc2, sd, p[e + 6], p[e + 7]);
      }
      l = l * al + ((sa + sb2) + (sc2 + sd));

      if (wg == 1) {
        // ---- branch 2: p2 (fp32) over its own score columns, row state to shared memory
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t rr[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(p[ch * 32 + e]);
          tmem_st32(sb + 64 + ch * 32, rr);
        }
        ms.h_a2[f][row] = al;
        ms.h_l2[f][row] = l;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ms.p2_ready[f]);
        continue;
      }

      // ---- branch 1: take branch 2's tile, choose c, keep D = O_1 - c O_2, write operands
      ok = mbar_wait(&ms.p2_ready[f], (j >> 1) & 1, abort_flag);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const float a2 = ms.h_a2[f][row];
      const float l2 = ms.h_l2[f][row];
      // target c = lambda l_1 / l_2 (sums including this tile); under max updates c follows
      // c a_1 / a_2, which leaves D unchanged; reset to the target when it leaves
      // [0.8, 1.25] times it (the row's first tile with a visible key always takes the
      // target: D and O_2 are still 0)
      const float cst = (WINDOW && !(l2 > 0.f)) ? lam : lam * __fdiv_rn(l, l2);  // exact ratio: identical branches give c = lambda
      float cn = cst, kc = 0.f;
      bool need = false;
      if (had) {
        const float cev = (al == a2) ? c : c * __fdividef(al, a2);
        const float ra = fabsf(cev), rt = fabsf(cst);
        const bool reset = !(ra >= 0.8f * rt && ra <= 1.25f * rt);
        cn = reset ? cst : cev;
        if (reset) kc = __fsub_rn(__fmul_rn(al, c), __fmul_rn(a2, cn));
        need = (al != 1.f) || (a2 != 1.f) || (kc != 0.f);
      }
      if (WINDOW || j > 0) {
        // the whole warp rescales (a row with nothing to do has al = a2 = 1, kc = 0)
        if (__any_sync(0xffffffffu, need)) {
          // D <- a_1 D + kc O_2, O_2 <- a_2 O_2 over all 128 output columns; the P.V MMAs
          // of the previous tile must have completed
          ok = mbar_wait(&ms.pv_done, (j - 1) & 1, abort_flag);
          if (!(ok = __all_sync(0xffffffffu, ok))) break;
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < 4; ++ch) {
            float dv[32], ov[32];
            tmem_ld32f(lane_addr + COL_D + ch * 32, dv);
            tmem_ld32f(lane_addr + COL_O2 + ch * 32, ov);
            tmem_wait_ld();
            uint32_t rd[32], ro[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              rd[e] = __float_as_uint(fmaf(kc, ov[e], al * dv[e]));
              ro[e] = __float_as_uint(a2 * ov[e]);
            }
            tmem_st32(lane_addr + COL_D + ch * 32, rd);
            tmem_st32(lane_addr + COL_O2 + ch * 32, ro);
          }
        }
      }
      c = cn;
      // operands: p1 - c p2 -> columns 0..31, p2 -> columns 32..63 (bf16 over S_1); the
      // statistics pass adds their remainders over the p2 columns of S_2 just read
      const float nc = -c;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float q2[32];
        tmem_ld32f(sb + 64 + ch * 32, q2);
        tmem_wait_ld();
        uint32_t pa[16], pb[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float w0, w1;
          ffma2(w0, w1, q2[e], q2[e + 1], nc, nc, p[ch * 32 + e], p[ch * 32 + e + 1]);
          pa[e / 2] = pack_bf16(w0, w1);
          pb[e / 2] = pack_bf16(q2[e], q2[e + 1]);
          if constexpr (STATS) {
            // the remainder x - hi(x) is exact in fp32; keep it in the registers of x
            p[ch * 32 + e] = w0 - __uint_as_float(pa[e / 2] << 16);
            p[ch * 32 + e + 1] = w1 - __uint_as_float(pa[e / 2] & 0xffff0000u);
            q2[e] -= __uint_as_float(pb[e / 2] << 16);
            q2[e + 1] -= __uint_as_float(pb[e / 2] & 0xffff0000u);
          }
        }
        tmem_st16(sb + ch * 16, pa);
        tmem_st16(sb + 32 + ch * 16, pb);
        if constexpr (STATS) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            pa[e / 2] = pack_bf16(p[ch * 32 + e], p[ch * 32 + e + 1]);
            pb[e / 2] = pack_bf16(q2[e], q2[e + 1]);
          }
          tmem_st16(sb + 64 + ch * 32, pa);
          tmem_st16(sb + 64 + ch * 32 + 16, pb);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ms.p_full[f]);
    }

    // ------------------------------- epilogue ----------------------------------------
    if (ok) ok = mbar_wait(&ms.o_full, 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    ms.ex_l[wg][row] = l;
    if (wg == 0) ms.ex_c[row] = c;
    bar_softmax();
    c = ms.ex_c[row];
    const float L1 = ms.ex_l[0][row], L2 = ms.ex_l[1][row];
    const float inv1 = 1.f / L1, inv2 = 1.f / L2;
    // o = D / l_1 + O_2 (c / l_1 - lambda / l_2); products rounded on their own so that
    // identical branches with lambda = 1 give exactly 0
    const float coef = __fsub_rn(__fmul_rn(c, inv1), __fmul_rn(lam, inv2));
    float y[64];
    float ss = 0.f;
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float dv[32], ov[32];
        tmem_ld32f(lane_addr + COL_D + wg * 64 + ch * 32, dv);
        tmem_ld32f(lane_addr + COL_O2 + wg * 64 + ch * 32, ov);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) y[ch * 32 + e] = __fmaf_rn(ov[e], coef, __fmul_rn(dv[e], inv1));
      }
#pragma unroll
      for (int e = 0; e < 64; ++e) ss = fmaf(y[e], y[e], ss);
    }
    if constexpr (STATS) {
      // dy over this thread's 64 channels (the output's layout)
      float gr[64];
      const int64_t dy_off = (int64_t)b * a.st_dys[0] + (int64_t)qi * a.st_dys[1] +
                             (int64_t)u * a.st_dys[2] + wg * 64;
      if (ok && qi < a.N && in_bounds(dy_off, 64, a.ext_st_dy, a.dev_status, a.dbg_status)) {
        const uint4* g4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.st_dy) + dy_off);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 w = g4[v];
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            gr[v * 8 + 2 * e] = __uint_as_float(wv[e] << 16);
            gr[v * 8 + 2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) gr[e] = 0.f;
      }
      float sdy = 0.f;
#pragma unroll
      for (int e = 0; e < 64; ++e) sdy = fmaf(gr[e], y[e], sdy);
      ms.ssx[wg][row] = ss;
      ms.ex_s[0][wg][row] = sdy;
      ms.ex_m[wg][row] = m;
      bar_softmax();
      const float m1 = ms.ex_m[0][row], m2 = ms.ex_m[1][row];
      if (a.apply_norm) {
        // out = s o / r with r^2 = mean(o^2) + eps and s = 1 - lambda_init, so the gradient
        // reaching o is s / r (dy - o (dy . o) / (n r^2)), n = 128
        const float r2 = (ms.ssx[0][row] + ms.ssx[1][row]) * (1.f / 128.f) + a.eps;
        const float f = (1.f - a.lambda_init[0]) * rsqrtf(r2);
        const float proj = (ms.ex_s[0][0][row] + ms.ex_s[0][1][row]) / (128.f * r2);
#pragma unroll
        for (int e = 0; e < 64; ++e) gr[e] = f * fmaf(-y[e], proj, gr[e]);
      }
      // delta_b = dO . O_b / l_b with the bf16 dO the backward's MMAs read (so that the
      // row's dS sums to zero over its operands), the dlambda share -dO . O_2 / l_2 with the
      // fp32 one; O_1 / l_1 = (D + c O_2) / l_1
      float e1 = 0.f, e2 = 0.f, e3 = 0.f;
      if (ok) {
        const float c1 = c * inv1;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          float dv[32], ov[32];
          tmem_ld32f(lane_addr + COL_D + wg * 64 + ch * 32, dv);
          tmem_ld32f(lane_addr + COL_O2 + wg * 64 + ch * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint32_t h = pack_bf16(gr[ch * 32 + e], gr[ch * 32 + e + 1]);
            const float g0 = __uint_as_float(h << 16), g1 = __uint_as_float(h & 0xffff0000u);
            const float o1a = __fmaf_rn(ov[e], c1, dv[e] * inv1), o1b = __fmaf_rn(ov[e + 1], c1, dv[e + 1] * inv1);
            const float o2a = ov[e] * inv2, o2b = ov[e + 1] * inv2;
            e1 = fmaf(g1, o1b, fmaf(g0, o1a, e1));
            e2 = fmaf(g1, o2b, fmaf(g0, o2a, e2));
            e3 = fmaf(gr[ch * 32 + e + 1], o2b, fmaf(gr[ch * 32 + e], o2a, e3));
          }
        }
      }
      ms.ex_s[1][wg][row] = e1;
      ms.ex_s[2][wg][row] = e2;
      ms.ex_s[3][wg][row] = e3;
      bar_softmax();
      if (ok && qi < a.N) {
        const int64_t do_off = (((int64_t)b * a.N + qi) * a.units + u) * 128 + wg * 64;
        if (in_bounds(do_off, 64, a.ext_st_do, a.dev_status, a.dbg_status)) {
          uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.st_do) + do_off);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            o4[v] = make_uint4(pack_bf16(gr[v * 8 + 0], gr[v * 8 + 1]), pack_bf16(gr[v * 8 + 2], gr[v * 8 + 3]),
                               pack_bf16(gr[v * 8 + 4], gr[v * 8 + 5]), pack_bf16(gr[v * 8 + 6], gr[v * 8 + 7]));
        }
        if (wg == 0) {
          const int64_t r = ((int64_t)b * a.units + u) * a.st_rows + qi;
          const int64_t rl = ((int64_t)b * a.units + u) * a.N + qi;
          if (in_bounds(r * 4, 4, a.ext_st, a.dev_status, a.dbg_status))
            *reinterpret_cast<float4*>(a.st + r * 4) =
                make_float4(m1 + log2f(L1), m2 + log2f(L2), ms.ex_s[1][0][row] + ms.ex_s[1][1][row],
                            ms.ex_s[2][0][row] + ms.ex_s[2][1][row]);
          if (in_bounds(rl, 1, a.ext_st_dl, a.dev_status, a.dbg_status))
            a.st_dl[rl] = -(ms.ex_s[3][0][row] + ms.ex_s[3][1][row]);
        }
      }
    } else {
      float sc = 1.f;
      ms.ssx[wg][row] = ss;
      bar_softmax();
      if (a.apply_norm)
        sc = rsqrtf((ms.ssx[0][row] + ms.ssx[1][row]) * (1.f / 128.f) + a.eps) *
             (1.f - a.lambda_init[0]);
      // (a variable-length tile reads its sequence back from shared memory, keeping the
      // registers of the key loop free)
      const int o_nq = VARLEN ? ms.seq_nq : a.N, o_b = VARLEN ? ms.seq_bc : b;
      const int o_q0 = VARLEN ? ms.seq_q0 : 0;
      const int64_t o_off = (int64_t)o_b * a.os[0] + (int64_t)(o_q0 + qi) * a.os[1] +
                            (int64_t)u * a.os[2] + wg * 64;
      if (ok && qi < o_nq && in_bounds(o_off, 64, a.ext_out, a.dev_status, a.dbg_status)) {
        __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.out) + o_off;
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

cudaError_t launch_prefill_v1(const PrefillArgs& a, cudaStream_t stream) {
  if (a.variant != DIFFATTN_V1 || a.d != 64) return cudaErrorNotSupported;
  TcMaps maps;
  // q, k viewed as [B, N, H, 128] (branch 1 in columns 0..63, branch 2 in 64..127) and v as
  // [B, N, H, 2d = 128]
  // a variable-length batch is one packed sequence of rows to the tensor maps
  const int rq = a.cu_q ? a.total_q : a.N, rk = a.cu_q ? a.total_k : a.Nk, nb = a.cu_q ? 1 : a.B;
  if (!make_map(&maps.q, a.q, 128, a.units, rq, nb, a.qs, BM)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, 128, a.units, rk, nb, a.ks, BN)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, 128, a.units, rk, nb, a.vs, BN)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const void* fns[4] = {(const void*)prefill_v1_kernel<false, false>, (const void*)prefill_v1_kernel<true, false>,
                          (const void*)prefill_v1_kernel<false, true>, (const void*)prefill_v1_kernel<true, true>};
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
    if (window) prefill_v1_kernel<true, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
    else prefill_v1_kernel<false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  } else {
    if (window) prefill_v1_kernel<true, false><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
    else prefill_v1_kernel<false, false><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  }
  return cudaGetLastError();
}

// The backward's statistics pass over the same tiles (fixed-length batches): st, st_dl,
// st_dy and st_do must be set; out is not written.
cudaError_t launch_prefill_v1_stats(const PrefillArgs& a, cudaStream_t stream) {
  if (a.variant != DIFFATTN_V1 || a.d != 64 || a.cu_q) return cudaErrorNotSupported;
  if (!a.st || !a.st_dl || !a.st_dy || !a.st_do) return cudaErrorInvalidValue;
  TcMaps maps;
  if (!make_map(&maps.q, a.q, 128, a.units, a.N, a.B, a.qs, BM)) return cudaErrorInvalidValue;
  if (!make_map(&maps.k, a.k, 128, a.units, a.Nk, a.B, a.ks, BN)) return cudaErrorInvalidValue;
  if (!make_map(&maps.v, a.v, 128, a.units, a.Nk, a.B, a.vs, BN)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const void* fns[2] = {(const void*)prefill_v1_kernel<false, false, true>,
                          (const void*)prefill_v1_kernel<true, false, true>};
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
    prefill_v1_kernel<true, false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  else
    prefill_v1_kernel<false, false, true><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace diffattn
