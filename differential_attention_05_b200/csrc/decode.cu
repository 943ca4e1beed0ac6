// decode.cu -- split-KV differential attention decode (V2: paired query heads over GQA).
//
// The KV cache is shared by both branches of every pair ("Differential Attention (V2)",
// "V1 vs V2": query heads doubled, KV heads unchanged, so decode loads the KV cache once).
// One block owns (batch b, KV head g, split s): it streams keys [s*T, (s+1)*T) of that KV
// head through a 3-stage cp.async ring (16-byte copies, fully coalesced 256-byte rows) and
// scores them for all 8 query heads of the group at once on the tensor cores
// (mma.sync m16n8k16: the 8 query heads are the M rows, padded to 16; keys are N; the
// head dimension is K). Every query head keeps its own running (max, sum, output); both
// branches of a pair are just two of those heads. P goes back into registers as the A
// operand of the P.V product, so nothing but the partial states leaves the chip.
//
// A second kernel merges the per-split states of each head,
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  O = sum_s o_s 2^(m_s - M) / L,
// and applies the difference per pair, out = O_(2p) - lambda_p * O_(2p+1)
// ("Differential Attention (V2)", The Concept: DiffAttn = (A_1 - lambda A_2) V).
#include "common.cuh"
#include "kernels.h"
#include "tma_host.cuh"

namespace diffattn {

namespace {
constexpr int D = 128;           // head dim
constexpr int G = 8;             // query heads per KV head
constexpr int CH = kDecodeChunk;  // keys per stage
constexpr int WARPS = 4;         // each warp: 16 keys of every chunk
constexpr int THREADS = WARPS * 32;
constexpr int STAGES = 3;
constexpr int ROW_BYTES = D * 2;
constexpr int TILE_BYTES = CH * ROW_BYTES;   // 16 KB
constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K + V
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;  // + alignment slack
constexpr int HALF_BYTES = CH * 128;         // one 64-column half of a tile: [64 rows x 128 B]
constexpr int CHUNKS16_PER_ROW = ROW_BYTES / 16;  // 16
static_assert(STAGES * STAGE_BYTES >= WARPS * (G * D + 2 * G) * 4, "merge scratch must fit");
}  // namespace

// A 64-key tile (K or V) in shared memory: two 64-column halves of [64 rows x 128 B] in
// the 128-byte swizzle TMA writes (16-byte chunk j of row r at chunk position j ^ (r % 8)),
// so the ldmatrix reads of 8 rows x 16 bytes hit 8 different bank groups.
__device__ __forceinline__ uint32_t swz(int row, int c16) {
  return (uint32_t)((c16 >> 3) * HALF_BYTES + row * 128 + (((c16 & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// C += A * B, m16n8k16, bf16 inputs, fp32 accumulate. Rows 8..15 of A are zero here
// (a1 = a3 = 0), so c2, c3 stay zero and are not used.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// MODE: the cache layout and how it is loaded.
//   kContig   contiguous cache [B, L, Hkv, d]: TMA boxes of 64 rows (zero fill past L);
//   kPagedTma page pool with pages of >= 8 tokens: TMA boxes of min(page size, 64) rows,
//             one per page of the chunk, each landing on a 1024-byte boundary;
//   kPagedCp  page pool with pages of 1, 2 or 4 tokens: 16-byte cp.async copies row by row.
// Rows past the entry's keys are zeroed in shared memory before use (V rows enter the P.V
// sums with weight 0, and 0 times a stale non-finite value would not be 0).
constexpr int kContig = 0, kPagedTma = 1, kPagedCp = 2;
template <int MODE>
__global__ void __launch_bounds__(THREADS, 2)
    decode_split_kernel(const __grid_constant__ TcMaps maps, DecodeArgs a) {
  constexpr bool PAGED = MODE != kContig;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full[STAGES];   // TMA modes: the chunk in stage s has landed
  __shared__ uint64_t bad_box[STAGES];  // kPagedTma: boxes of the chunk in stage s not loaded
  __shared__ int abort_flag;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;  // mma fragment row / column-pair index

  // device-side lengths are clamped into [0, L] so a bad value cannot read past the cache
  const int kv_len = a.kv_len ? min(max(a.kv_len[b], 0), a.L) : a.L;
  const int t_begin = split * a.split_len;
  const int t_end = min(t_begin + a.split_len, kv_len);
  const int n_chunks = t_end > t_begin ? (t_end - t_begin + CH - 1) / CH : 0;

  // paged cache: this entry's row of the block table; the page stride replaces the batch one
  const int64_t boff = PAGED ? 0 : b * a.kvs[0];
  const __nv_bfloat16* kbase =
      static_cast<const __nv_bfloat16*>(a.k) + boff + (int64_t)g * a.kvs[2];
  const __nv_bfloat16* vbase =
      static_cast<const __nv_bfloat16*>(a.v) + boff + (int64_t)g * a.kvs[2];
  bool bad_page = false;  // a block-table entry outside the pool: its rows read as zero

  // Each thread copies the same ROWS_T rows of every chunk, (tid / CHUNKS16_PER_ROW) + RSTEP i, for K
  // and for V. With a paged cache their page ids are fetched one chunk ahead (fetch_ids),
  // so the table reads overlap the work on the current chunk.
  constexpr int RSTEP = THREADS / CHUNKS16_PER_ROW;               // rows covered by one pass of the block
  constexpr int ROWS_T = CH / RSTEP;                   // rows per thread and tensor
  static_assert(THREADS % CHUNKS16_PER_ROW == 0 && CH % RSTEP == 0, "copy layout");
  int pid[MODE == kPagedCp ? ROWS_T : 1];
  auto fetch_ids = [&](int c) {
    if constexpr (MODE == kPagedCp) {
      const int tok0 = t_begin + c * CH + tid / CHUNKS16_PER_ROW;
#pragma unroll
      for (int i = 0; i < ROWS_T; ++i) {
        const int tok = tok0 + RSTEP * i;
        const int64_t bi = (int64_t)b * a.bt_stride + (tok >> a.page_shift);
        pid[i] = (tok < t_end && in_bounds(bi, 1, a.ext_bt, a.dev_status, a.dbg_status))
                     ? __ldg(a.block_table + bi) : 0;
      }
    }
  };

  // kPagedCp: issue the copies of chunk c into stage c % STAGES (zero-fill past t_end)
  auto load_chunk_cp = [&](int c) {
    uint8_t* st = smem + (c % STAGES) * STAGE_BYTES;
    const int tok0 = t_begin + c * CH;
#pragma unroll
    for (int it = 0; it < (2 * CH * CHUNKS16_PER_ROW) / THREADS; ++it) {
      const int idx = tid + it * THREADS;
      const int tensor = idx / (CH * CHUNKS16_PER_ROW);
      const int rem = idx % (CH * CHUNKS16_PER_ROW);
      const int row = rem / CHUNKS16_PER_ROW, c16 = rem % CHUNKS16_PER_ROW;  // row = tid / CHUNKS16_PER_ROW + RSTEP (it % ROWS_T)
      const int tok = tok0 + row;
      bool ok = tok < t_end;
      int64_t roff;
      if constexpr (PAGED) {
        const int id = pid[it % ROWS_T];
        if ((unsigned)id >= (unsigned)a.num_pages) {
          bad_page = bad_page || ok;
          ok = false;
        }
        roff = (int64_t)id * a.kvs[0] + (int64_t)(tok & ((1 << a.page_shift) - 1)) * a.kvs[1];
      } else {
        roff = (int64_t)tok * a.kvs[1];
      }
      const int64_t soff = boff + (int64_t)g * a.kvs[2] + (ok ? roff : 0) + c16 * 8;
      ok = ok && in_bounds(soff, 8, a.ext_kv, a.dev_status, a.dbg_status);
      const __nv_bfloat16* src = (tensor ? vbase : kbase) + (ok ? roff : 0) + c16 * 8;
      cp_async_16(st + tensor * TILE_BYTES + swz(row, c16), src, ok ? 16u : 0u);
    }
  };

  // kPagedTma: lane i % 32 of warp 0 reads the page ids of box i of a chunk one chunk ahead
  // of its copies (fetch_ids_tma), so the table reads overlap the work on the current chunk;
  // -1 marks a box wholly past t_end
  int pid_t[2] = {-1, -1};
  auto fetch_ids_tma = [&](int c) {
    if constexpr (MODE == kPagedTma) {
      const int pshift = min(a.page_shift, 6), pr = 1 << pshift, nbox = CH >> pshift;
      const int tok0 = t_begin + c * CH;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = lane + 32 * r;
        const int t = tok0 + i * pr;
        pid_t[r] = -1;
        if (i < nbox && t < t_end) {
          const int64_t bi = (int64_t)b * a.bt_stride + (t >> a.page_shift);
          pid_t[r] = in_bounds(bi, 1, a.ext_bt, a.dev_status, a.dbg_status) ? __ldg(a.block_table + bi)
                                                                             : a.num_pages;
        }
      }
    }
  };

  // TMA modes: warp 0 issues the copies of chunk c into stage c % STAGES. Paged: box i
  // (rows i * pr .. of the chunk) is one page's run of pr tokens; lane i % 32 issues its
  // copies with the page id fetched before. A box wholly past t_end is not loaded (zeroed
  // after the wait), nor is one whose page id lies outside the pool (zeroed and reported).
  auto load_chunk_tma = [&](int c) {
    uint8_t* st = smem + (c % STAGES) * STAGE_BYTES;
    uint64_t* bar = &full[c % STAGES];
    const int tok0 = t_begin + c * CH;
    if constexpr (MODE == kContig) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, 2 * TILE_BYTES);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_4d(st + hf * HALF_BYTES, &maps.k, bar, 64 * hf, g, tok0, b);
          tma_load_4d(st + TILE_BYTES + hf * HALF_BYTES, &maps.v, bar, 64 * hf, g, tok0, b);
        }
      }
    } else if constexpr (MODE == kPagedTma) {
      const int pr = 1 << min(a.page_shift, 6), nbox = CH / pr;
      const int pmask = (1 << a.page_shift) - 1;
      int ids[2];
      bool load[2] = {false, false}, bad[2] = {false, false};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = lane + 32 * r;
        if (i < nbox && tok0 + i * pr < t_end) {
          ids[r] = pid_t[r];
          load[r] = (unsigned)ids[r] < (unsigned)a.num_pages;
          bad[r] = !load[r];
        }
      }
      const uint32_t lmask0 = __ballot_sync(0xffffffffu, load[0]), lmask1 = __ballot_sync(0xffffffffu, load[1]);
      const uint32_t bmask0 = __ballot_sync(0xffffffffu, bad[0]), bmask1 = __ballot_sync(0xffffffffu, bad[1]);
      if (lane == 0) {
        bad_box[c % STAGES] = (uint64_t)bmask0 | ((uint64_t)bmask1 << 32);
        const int nl = __popc(lmask0) + __popc(lmask1);
        mbar_arrive_expect_tx(bar, (uint32_t)(nl * pr * 128 * 4));  // K and V, both halves
      }
      __syncwarp();
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (!load[r]) continue;
        const int i = lane + 32 * r;
        const int row = (tok0 + i * pr) & pmask;  // first row of the run inside its page
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_4d(st + hf * HALF_BYTES + i * pr * 128, &maps.k, bar, 64 * hf, g, row, ids[r]);
          tma_load_4d(st + TILE_BYTES + hf * HALF_BYTES + i * pr * 128, &maps.v, bar, 64 * hf, g, row, ids[r]);
        }
      }
      if (bmask0 | bmask1) bad_page = true;
    }
  };

  // TMA modes, after chunk c has landed: zero the V rows of the chunk past t_end (and, for a
  // page outside the pool, its K and V rows), so that they add exactly 0 to the P.V sums
  auto zero_rows = [&](int c) {
    if constexpr (MODE != kPagedCp) {
      uint8_t* st = smem + (c % STAGES) * STAGE_BYTES;
      const int valid = t_end - (t_begin + c * CH);  // rows < valid are keys of the entry
      uint64_t bad = 0;
      int pr = CH;
      if constexpr (MODE == kPagedTma) {
        bad = bad_box[c % STAGES];
        pr = 1 << min(a.page_shift, 6);
      }
      if (valid < CH || bad) {
        for (int idx = tid; idx < 2 * CH * CHUNKS16_PER_ROW; idx += THREADS) {
          const int tensor = idx / (CH * CHUNKS16_PER_ROW);
          const int rem = idx % (CH * CHUNKS16_PER_ROW);
          const int row = rem / CHUNKS16_PER_ROW, c16 = rem % CHUNKS16_PER_ROW;
          const bool bad_row = (bad >> (row / pr)) & 1;
          if ((tensor == 1 && row >= valid) || bad_row)
            *reinterpret_cast<uint4*>(st + tensor * TILE_BYTES + swz(row, c16)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();  // before a later TMA copy rewrites the stage
      }
    }
  };

  // Q fragments of the 8 heads (A operand, rows 0..7), all 8 k-steps of d = 128
  uint32_t qa[8][2];
  {
    const int64_t q_off = b * a.qs[0] + (int64_t)(g * G + gq) * a.qs[1];
    const bool q_ok = in_bounds(q_off, D, a.ext_q, a.dev_status, a.dbg_status);
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(a.q) + q_off);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = q_ok ? q32[(ks * 16 + 2 * tq) / 2] : 0u;
      qa[ks][1] = q_ok ? q32[(ks * 16 + 8 + 2 * tq) / 2] : 0u;
    }
  }

  const float sl2 = 1.4426950408889634f / sqrtf((float)D);  // log2(e) / sqrt(d)
  float m = -INFINITY, l = 0.f;                              // head gq, log2 domain
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  if constexpr (MODE != kPagedCp) {
    if (tid == 0) {
      for (int st = 0; st < STAGES; ++st) mbar_init(&full[st], 1);
      abort_flag = 0;
      fence_barrier_init();
    }
    __syncthreads();
  }
  int issued = 0;  // TMA modes: chunks whose copies were issued
#pragma unroll
  for (int c = 0; c < STAGES - 1; ++c) {
    if constexpr (MODE == kPagedCp) {
      if (c < n_chunks) {
        fetch_ids(c);
        load_chunk_cp(c);
      }
      cp_async_commit();
    } else if (c < n_chunks) {
      if (warp == 0) {
        fetch_ids_tma(c);
        load_chunk_tma(c);
      }
      issued = c + 1;
    }
  }
  if constexpr (MODE == kPagedCp) {
    if (STAGES - 1 < n_chunks) fetch_ids(STAGES - 1);
  } else {
    if (STAGES - 1 < n_chunks && warp == 0) fetch_ids_tma(STAGES - 1);
  }

  for (int c = 0; c < n_chunks; ++c) {
    if constexpr (MODE == kPagedCp) {
      if (c + STAGES - 1 < n_chunks) {
        load_chunk_cp(c + STAGES - 1);
        if (c + STAGES < n_chunks) fetch_ids(c + STAGES);
      }
      cp_async_commit();
      cp_async_wait<STAGES - 1>();
      __syncthreads();
    } else {
      // stage (c + 2) % STAGES was released by the __syncthreads ending iteration c - 1
      if (c + STAGES - 1 < n_chunks) {
        if (warp == 0) {
          load_chunk_tma(c + STAGES - 1);
          if (c + STAGES < n_chunks) fetch_ids_tma(c + STAGES);
        }
        issued = c + STAGES;
      }
      const bool ok = mbar_wait(&full[c % STAGES], (c / STAGES) & 1, &abort_flag);
      if (!__syncthreads_and(ok)) {
        // a copy that never landed: let the ones in flight finish before the shared memory
        // is reused below, and report
        if (tid == 0) {
          for (int cc = c; cc < issued; ++cc) mbar_wait_drain(&full[cc % STAGES], (cc / STAGES) & 1);
          report_status(a.dev_status, DIFFATTN_ERR_TIMEOUT);
        }
        __syncthreads();
        break;
      }
      zero_rows(c);
      __syncthreads();
    }

    const uint32_t kst = smem_u32(smem + (c % STAGES) * STAGE_BYTES);
    const uint32_t vst = kst + TILE_BYTES;

    // S = Q K^T for this warp's 16 keys (two n-tiles of 8 keys)
    float s[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int mat = lane >> 3;
      const int row = warp * 16 + (mat >> 1) * 8 + (lane & 7);
      const int c16 = 2 * ks + (mat & 1);
      uint32_t b00, b01, b10, b11;
      ldsm_x4(kst + swz(row, c16), b00, b01, b10, b11);
      mma16816(s[0], qa[ks][0], qa[ks][1], b00, b01);
      mma16816(s[1], qa[ks][0], qa[ks][1], b10, b11);
    }

    // online softmax for head gq over keys warp*16 + {n*8 + 2tq, +1}
    const int tok0 = t_begin + c * CH + warp * 16;
    float x[4];
    float mx = -INFINITY;
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = tok0 + n * 8 + 2 * tq + e;
        const float v = tok < t_end ? s[n][e] * sl2 : -INFINITY;
        x[n * 2 + e] = v;
        mx = fmaxf(mx, v);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mn = fmaxf(m, mx);
    const float alpha = (m == -INFINITY) ? 0.f : ex2(m - mn);
    float p[4];
    float ps = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = (x[e] == -INFINITY) ? 0.f : ex2(x[e] - mn);
      ps += p[e];
    }
    l = l * alpha + ps;
    m = mn;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= alpha;
      o[n][1] *= alpha;
    }

    // O += P V : P (rows = heads, k = this warp's 16 keys) straight from registers
    const uint32_t pa0 = pack_bf16(p[0], p[1]);
    const uint32_t pa2 = pack_bf16(p[2], p[3]);
#pragma unroll
    for (int np = 0; np < 8; ++np) {
      const int mat = lane >> 3;
      const int row = warp * 16 + (mat & 1) * 8 + (lane & 7);
      const int c16 = 2 * np + (mat >> 1);
      uint32_t b0a, b1a, b0b, b1b;
      ldsm_x4_t(vst + swz(row, c16), b0a, b1a, b0b, b1b);
      mma16816(o[2 * np], pa0, pa2, b0a, b1a);
      mma16816(o[2 * np + 1], pa0, pa2, b0b, b1b);
    }
    __syncthreads();  // stage c % STAGES is refilled on the next iteration
  }
  if constexpr (MODE == kPagedCp) cp_async_wait<0>();
  __syncthreads();
  if (bad_page) report_status(a.dev_status, DIFFATTN_ERR_INVALID_ARG);

  // merge the 4 warps' states of each head through shared memory
  float* sm_o = reinterpret_cast<float*>(smem);      // [WARPS][G][D]
  float* sm_ml = sm_o + WARPS * G * D;               // [WARPS][G][2]
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    sm_o[(warp * G + gq) * D + n * 8 + 2 * tq] = o[n][0];
    sm_o[(warp * G + gq) * D + n * 8 + 2 * tq + 1] = o[n][1];
  }
  if (tq == 0) {
    sm_ml[(warp * G + gq) * 2 + 0] = m;
    sm_ml[(warp * G + gq) * 2 + 1] = l;
  }
  __syncthreads();
  {
    const int h = tid / 16, c0 = (tid % 16) * 8;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, sm_ml[(w * G + h) * 2]);
    float f[WARPS];
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float mw = sm_ml[(w * G + h) * 2];
      f[w] = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      L += sm_ml[(w * G + h) * 2 + 1] * f[w];
    }
    const int hq = g * G + h;
    const int64_t rec = ((int64_t)b * a.Hq + hq) * a.splits + split;
    float4* dst = reinterpret_cast<float4*>(a.ws_o + rec * D + c0);
    const bool w_ok = in_bounds(rec * D + c0, 8, a.ext_ws_o, a.dev_status, a.dbg_status);
#pragma unroll
    for (int v4 = 0; v4 < 2 && w_ok; ++v4) {
      float r[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) acc += sm_o[(w * G + h) * D + c0 + v4 * 4 + e] * f[w];
        r[e] = acc;
      }
      dst[v4] = make_float4(r[0], r[1], r[2], r[3]);
    }
    if ((tid % 16) == 0 && in_bounds(rec * 2, 2, a.ext_ws_ml, a.dev_status, a.dbg_status)) {
      a.ws_ml[rec * 2 + 0] = M;
      a.ws_ml[rec * 2 + 1] = L;
    }
  }
}

__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeArgs a) {
  const int p = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  float res[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int hq = 2 * p + e;
    const int64_t rec0 = ((int64_t)b * a.Hq + hq) * a.splits;
    if (!in_bounds(rec0 * 2, 2 * (int64_t)a.splits, a.ext_ws_ml, a.dev_status, a.dbg_status) ||
        !in_bounds(rec0 * D, (int64_t)a.splits * D, a.ext_ws_o, a.dev_status, a.dbg_status)) {
      res[e] = 0.f;
      continue;
    }
    float M = -INFINITY;
    for (int s = 0; s < a.splits; ++s) M = fmaxf(M, a.ws_ml[(rec0 + s) * 2]);
    float L = 0.f, O = 0.f;
    for (int s = 0; s < a.splits; ++s) {
      const float ms = a.ws_ml[(rec0 + s) * 2];
      if (ms == -INFINITY) continue;
      const float f = ex2(ms - M);
      L += a.ws_ml[(rec0 + s) * 2 + 1] * f;
      O += a.ws_o[(rec0 + s) * D + c] * f;
    }
    res[e] = L > 0.f ? O / L : 0.f;
  }
  const float y = res[0] - a.lambda[p] * res[1];
  const int64_t o_off = b * a.os[0] + (int64_t)p * a.os[1];
  if (in_bounds(o_off + c, 1, a.ext_out, a.dev_status, a.dbg_status))
    static_cast<__nv_bfloat16*>(a.out)[o_off + c] = __float2bfloat16_rn(y);
}

int decode_default_splits(int B, int L, int Hkv) {
  const int pairs = B * Hkv;
  int s = (L + 4095) / 4096;
  const int min_blocks = 2 * 148 * 2;
  if (pairs > 0 && pairs * s < min_blocks) s = (min_blocks + pairs - 1) / pairs;
  const int max_s = (L + CH - 1) / CH;
  if (s > max_s) s = max_s;
  return s < 1 ? 1 : s;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const void* fns[3] = {(const void*)decode_split_kernel<kContig>, (const void*)decode_split_kernel<kPagedTma>,
                          (const void*)decode_split_kernel<kPagedCp>};
    for (const void* fn : fns) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    if (dev < 64) attr_set[dev] = true;
  }
  // tensor maps: K and V as {d, Hkv, rows, batch entries} (contiguous) or {d, Hkv, page size,
  // pages} (pool), 64-column boxes of 64 rows (contiguous) or of one page's run of up to 64
  // rows, 128-byte swizzle, zero fill outside the tensor
  TcMaps maps = {};
  const int ps = 1 << a.page_shift;
  const int mode = !a.block_table ? kContig : (ps >= 8 ? kPagedTma : kPagedCp);
  if (mode == kContig) {
    if (!make_map(&maps.k, a.k, D, a.Hkv, a.L, a.B, a.kvs, CH)) return cudaErrorInvalidValue;
    if (!make_map(&maps.v, a.v, D, a.Hkv, a.L, a.B, a.kvs, CH)) return cudaErrorInvalidValue;
  } else if (mode == kPagedTma) {
    const int pr = ps < CH ? ps : CH;
    if (!make_map(&maps.k, a.k, D, a.Hkv, ps, a.num_pages, a.kvs, pr)) return cudaErrorInvalidValue;
    if (!make_map(&maps.v, a.v, D, a.Hkv, ps, a.num_pages, a.kvs, pr)) return cudaErrorInvalidValue;
  }
  dim3 grid(a.splits, a.Hkv, a.B);
  if (mode == kContig)
    decode_split_kernel<kContig><<<grid, THREADS, SMEM_BYTES, stream>>>(maps, a);
  else if (mode == kPagedTma)
    decode_split_kernel<kPagedTma><<<grid, THREADS, SMEM_BYTES, stream>>>(maps, a);
  else
    decode_split_kernel<kPagedCp><<<grid, THREADS, SMEM_BYTES, stream>>>(maps, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid2(a.Hq / 2, a.B);
  decode_combine_kernel<<<grid2, D, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace diffattn
