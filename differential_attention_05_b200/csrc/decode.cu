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
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES;
constexpr int CHUNKS16_PER_ROW = ROW_BYTES / 16;  // 16
static_assert(SMEM_BYTES >= WARPS * (G * D + 2 * G) * 4, "merge scratch must fit");
}  // namespace

__device__ __forceinline__ uint32_t swz(int row, int c16) {
  return (uint32_t)(row * ROW_BYTES + ((c16 ^ (row & 7)) << 4));
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

// PAGED: the cache is a page pool addressed through a block table (DecodeArgs); the
// contiguous instantiation has none of that code.
template <bool PAGED>
__global__ void __launch_bounds__(THREADS, 2) decode_split_kernel(DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
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
  int pid[PAGED ? ROWS_T : 1];
  auto fetch_ids = [&](int c) {
    if constexpr (PAGED) {
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

  // issue the copies of chunk c into stage c % STAGES (zero-fill past t_end)
  auto load_chunk = [&](int c) {
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

#pragma unroll
  for (int c = 0; c < STAGES - 1; ++c) {
    if (c < n_chunks) {
      fetch_ids(c);
      load_chunk(c);
    }
    cp_async_commit();
  }
  if (STAGES - 1 < n_chunks) fetch_ids(STAGES - 1);

  for (int c = 0; c < n_chunks; ++c) {
    if (c + STAGES - 1 < n_chunks) {
      load_chunk(c + STAGES - 1);
      if (c + STAGES < n_chunks) fetch_ids(c + STAGES);
    }
    cp_async_commit();
    cp_async_wait<STAGES - 1>();
    __syncthreads();

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
  cp_async_wait<0>();
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
    e = cudaFuncSetAttribute(decode_split_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_split_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  dim3 grid(a.splits, a.Hkv, a.B);
  if (a.block_table)
    decode_split_kernel<true><<<grid, THREADS, SMEM_BYTES, stream>>>(a);
  else
    decode_split_kernel<false><<<grid, THREADS, SMEM_BYTES, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid2(a.Hq / 2, a.B);
  decode_combine_kernel<<<grid2, D, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace diffattn
