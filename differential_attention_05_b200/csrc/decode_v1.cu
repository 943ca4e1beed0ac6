// decode_v1.cu -- split-KV differential attention decode for V1 (two branches with their
// own cached keys K_1, K_2 of width d = 64 and one cached value row of width 2d = 128).
//
// "Differential Attention (V2)", "V1 vs V2": V1 decode as the pages describe it loads the
// value cache twice (one attention call per branch). Here one block owns (batch b, head h,
// split s) and streams keys [s*T, (s+1)*T) of that head through a 3-stage cp.async ring;
// every cached (K_1 | K_2, V) row is read from memory once and serves both branches.
// Per key and head the work is 2 x 64 multiply-adds for the scores and 2 x 128 for P.V
// against 512 bytes of cache, 1.5 FLOP per byte: the FMA pipe keeps up with HBM, so this
// kernel runs on the CUDA cores in fp32 (no bf16 rounding of the probabilities at all).
//   * scores: thread t scores key t % 64 of the chunk for branch t / 64 from shared
//     memory (16-byte loads, rows XOR-swizzled so a warp's loads are conflict-free);
//   * online softmax per branch in the log2 domain (max and sum over the branch's two
//     warps through shared memory), probabilities to shared memory;
//   * P.V: thread t accumulates value columns 2(t % 64), +1 of both branches over key half
//     t / 64 of every chunk; the halves are added once at the end of the split.
// A second kernel merges the per-split states of each (b, h) and forms
//   o = O_1/l_1 - lambda O_2/l_2,  o <- o / sqrt(mean(o^2) + eps) * (1 - lambda_init)
// ("Differential Attention (V2)", The Concept, "The difference idea"; "V1 vs V2" and Key
//  Terms, per-head RMSNorm).
#include "common.cuh"
#include "kernels.h"

namespace diffattn {

namespace {
constexpr int D1 = 64;                 // branch width
constexpr int DV = 2 * D1;             // value width
constexpr int CH = kDecodeChunk;       // keys per stage (64)
constexpr int THREADS = 128;
constexpr int STAGES = 3;
constexpr int ROW_BYTES = 256;         // one cached K row (K_1 | K_2) or V row, bf16
constexpr int TILE_BYTES = CH * ROW_BYTES;   // 16 KB
constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K + V
constexpr int RING_BYTES = STAGES * STAGE_BYTES;
constexpr int C16 = ROW_BYTES / 16;    // 16-byte chunks per row
// shared scratch after the ring: probabilities [2][CH], branch maxima / sums [2 warps][2]
constexpr int SCRATCH_BYTES = 2 * CH * 4 + 2 * 2 * 4 * 2;
constexpr int SMEM_BYTES = RING_BYTES + SCRATCH_BYTES;
static_assert(RING_BYTES >= THREADS * 4 * 4, "end-of-split exchange must fit in the ring");
}  // namespace

// byte offset of 16-byte chunk c16 of row `row` in a swizzled [CH x 256 B] tile
__device__ __forceinline__ uint32_t swz_v1(int row, int c16) {
  return (uint32_t)(row * ROW_BYTES + ((c16 ^ (row & 15)) << 4));
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// PAGED: the cache is a page pool addressed through a block table (DecodeArgs); the
// contiguous instantiation has none of that code.
template <bool PAGED>
__global__ void __launch_bounds__(THREADS, 2) decode_v1_split_kernel(DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  float* ps = reinterpret_cast<float*>(smem + RING_BYTES);  // [2][CH] probabilities
  float* red = ps + 2 * CH;                                   // [branch][warp of branch][max, sum]
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31;
  const int br = tid >> 6;          // branch this thread scores
  const int key = tid & 63;         // key of the chunk it scores
  const int wb = (tid >> 5) & 1;    // warp index within the branch
  const int cp = tid & 63;          // value column pair it accumulates
  const int kh = tid >> 6;          // key half it accumulates

  // device-side lengths are clamped into [0, L] so a bad value cannot read past the cache
  const int kv_len = a.kv_len ? min(max(a.kv_len[b], 0), a.L) : a.L;
  const int t_begin = split * a.split_len;
  const int t_end = min(t_begin + a.split_len, kv_len);
  const int n_chunks = t_end > t_begin ? (t_end - t_begin + CH - 1) / CH : 0;

  // paged cache: this entry's row of the block table; the page stride replaces the batch one
  const int64_t boff = PAGED ? 0 : b * a.kvs[0];
  const __nv_bfloat16* kbase =
      static_cast<const __nv_bfloat16*>(a.k) + boff + (int64_t)h * a.kvs[2];
  const __nv_bfloat16* vbase =
      static_cast<const __nv_bfloat16*>(a.v) + boff + (int64_t)h * a.kvs[2];
  bool bad_page = false;  // a block-table entry outside the pool: its rows read as zero

  // Each thread copies the same ROWS_T rows of every chunk, (tid / C16) + RSTEP i, for K
  // and for V. With a paged cache their page ids are fetched one chunk ahead (fetch_ids),
  // so the table reads overlap the work on the current chunk.
  constexpr int RSTEP = THREADS / C16;               // rows covered by one pass of the block
  constexpr int ROWS_T = CH / RSTEP;                   // rows per thread and tensor
  static_assert(THREADS % C16 == 0 && CH % RSTEP == 0, "copy layout");
  int pid[PAGED ? ROWS_T : 1];
  auto fetch_ids = [&](int c) {
    if constexpr (PAGED) {
      const int tok0 = t_begin + c * CH + tid / C16;
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
    for (int it = 0; it < (2 * CH * C16) / THREADS; ++it) {
      const int idx = tid + it * THREADS;
      const int tensor = idx / (CH * C16);
      const int rem = idx % (CH * C16);
      const int row = rem / C16, c16 = rem % C16;  // row = tid / C16 + RSTEP (it % ROWS_T)
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
      const int64_t soff = boff + (int64_t)h * a.kvs[2] + (ok ? roff : 0) + c16 * 8;
      ok = ok && in_bounds(soff, 8, a.ext_kv, a.dev_status, a.dbg_status);
      const __nv_bfloat16* src = (tensor ? vbase : kbase) + (ok ? roff : 0) + c16 * 8;
      cp_async_16(st + tensor * TILE_BYTES + swz_v1(row, c16), src, ok ? 16u : 0u);
    }
  };

  // this thread's query branch (64 values) in fp32
  float q[D1];
  {
    const int64_t q_off = b * a.qs[0] + (int64_t)h * a.qs[1] + br * D1;
    const bool q_ok = in_bounds(q_off, D1, a.ext_q, a.dev_status, a.dbg_status);
    const uint4* q4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + q_off);
#pragma unroll
    for (int i = 0; i < D1 / 8; ++i) {
      const uint4 w = q_ok ? q4[i] : make_uint4(0u, 0u, 0u, 0u);
      q[8 * i + 0] = bf16lo(w.x); q[8 * i + 1] = bf16hi(w.x);
      q[8 * i + 2] = bf16lo(w.y); q[8 * i + 3] = bf16hi(w.y);
      q[8 * i + 4] = bf16lo(w.z); q[8 * i + 5] = bf16hi(w.z);
      q[8 * i + 6] = bf16lo(w.w); q[8 * i + 7] = bf16hi(w.w);
    }
  }

  const float sl2 = 1.4426950408889634f / sqrtf((float)D1);  // log2(e) / sqrt(d)
  float m1 = -INFINITY, m2 = -INFINITY, l1 = 0.f, l2 = 0.f;  // both branches, log2 domain
  float o1x = 0.f, o1y = 0.f, o2x = 0.f, o2y = 0.f;          // columns 2cp, 2cp+1

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

    const uint8_t* kst = smem + (c % STAGES) * STAGE_BYTES;
    const uint8_t* vst = kst + TILE_BYTES;

    // score of (branch br, key) in the log2 domain
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
    for (int i = 0; i < D1 / 8; ++i) {
      const uint4 w = *reinterpret_cast<const uint4*>(kst + swz_v1(key, br * 8 + i));
      s0 = fmaf(q[8 * i + 0], bf16lo(w.x), s0); s1 = fmaf(q[8 * i + 1], bf16hi(w.x), s1);
      s2 = fmaf(q[8 * i + 2], bf16lo(w.y), s2); s3 = fmaf(q[8 * i + 3], bf16hi(w.y), s3);
      s0 = fmaf(q[8 * i + 4], bf16lo(w.z), s0); s1 = fmaf(q[8 * i + 5], bf16hi(w.z), s1);
      s2 = fmaf(q[8 * i + 6], bf16lo(w.w), s2); s3 = fmaf(q[8 * i + 7], bf16hi(w.w), s3);
    }
    const int tok = t_begin + c * CH + key;
    const float x = tok < t_end ? ((s0 + s1) + (s2 + s3)) * sl2 : -INFINITY;

    // the branch's chunk maximum over its two warps
    const float wm = warp_max(x);
    if (lane == 0) red[(br * 2 + wb) * 2] = wm;
    __syncthreads();
    const float cm1 = fmaxf(red[0], red[2]), cm2 = fmaxf(red[4], red[6]);
    const float n1 = fmaxf(m1, cm1), n2 = fmaxf(m2, cm2);
    // chunks wholly past t_end do not occur (n_chunks stops at t_end), so n1, n2 > -inf
    const float al1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - n1);
    const float al2 = (m2 == -INFINITY) ? 0.f : ex2(m2 - n2);
    const float p = (x == -INFINITY) ? 0.f : ex2(x - (br ? n2 : n1));
    ps[br * CH + key] = p;
    const float wsum = warp_sum(p);
    if (lane == 0) red[(br * 2 + wb) * 2 + 1] = wsum;
    __syncthreads();
    l1 = l1 * al1 + (red[1] + red[3]);
    l2 = l2 * al2 + (red[5] + red[7]);
    m1 = n1;
    m2 = n2;

    // P.V over this thread's key half, value columns 2cp, 2cp+1, both branches
    o1x *= al1; o1y *= al1; o2x *= al2; o2y *= al2;
#pragma unroll 8
    for (int e = 0; e < CH / 2; ++e) {
      const int k = kh * (CH / 2) + e;
      const uint32_t w =
          *reinterpret_cast<const uint32_t*>(vst + swz_v1(k, cp >> 2) + (cp & 3) * 4);
      const float vx = bf16lo(w), vy = bf16hi(w);
      const float p1 = ps[k], p2 = ps[CH + k];
      o1x = fmaf(p1, vx, o1x); o1y = fmaf(p1, vy, o1y);
      o2x = fmaf(p2, vx, o2x); o2y = fmaf(p2, vy, o2y);
    }
    __syncthreads();  // the stage and the scratch are rewritten next iteration
  }
  cp_async_wait<0>();
  if (bad_page) report_status(a.dev_status, DIFFATTN_ERR_INVALID_ARG);

  // add the two key halves and write the split's partial state:
  // ws_o[((b*H + h)*splits + s)*2 + branch][128], ws_ml[...][2] = (m, l)
  float* ex = reinterpret_cast<float*>(smem);
  __syncthreads();
  if (kh == 1) {
    ex[cp * 4 + 0] = o1x; ex[cp * 4 + 1] = o1y; ex[cp * 4 + 2] = o2x; ex[cp * 4 + 3] = o2y;
  }
  __syncthreads();
  if (kh == 0) {
    o1x += ex[cp * 4 + 0]; o1y += ex[cp * 4 + 1]; o2x += ex[cp * 4 + 2]; o2y += ex[cp * 4 + 3];
    const size_t rec = ((size_t)(b * gridDim.y + h) * gridDim.x + split) * 2;
    float* w1 = a.ws_o + rec * DV;
    float* w2 = w1 + DV;
    if (in_bounds((int64_t)rec * DV + 2 * cp, DV + 2, a.ext_ws_o, a.dev_status, a.dbg_status)) {
      w1[2 * cp] = o1x; w1[2 * cp + 1] = o1y;
      w2[2 * cp] = o2x; w2[2 * cp + 1] = o2y;
    }
    if (cp == 0 && in_bounds((int64_t)rec * 2, 4, a.ext_ws_ml, a.dev_status, a.dbg_status)) {
      a.ws_ml[rec * 2 + 0] = m1; a.ws_ml[rec * 2 + 1] = l1;
      a.ws_ml[rec * 2 + 2] = m2; a.ws_ml[rec * 2 + 3] = l2;
    }
  }
}

// One block of 128 threads per (b, h): thread c owns value column c.
__global__ void __launch_bounds__(DV) decode_v1_combine_kernel(DecodeArgs a) {
  __shared__ float red[4];
  const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  const int S = a.splits;
  const size_t rec0 = (size_t)(b * gridDim.x + h) * S * 2;
  const bool r_ok = in_bounds((int64_t)rec0 * 2, 4 * (int64_t)S, a.ext_ws_ml, a.dev_status, a.dbg_status) &&
                    in_bounds((int64_t)rec0 * DV, 2 * (int64_t)S * DV, a.ext_ws_o, a.dev_status, a.dbg_status);
  float M1 = -INFINITY, M2 = -INFINITY;
  for (int s = 0; s < S && r_ok; ++s) {
    M1 = fmaxf(M1, a.ws_ml[(rec0 + 2 * s) * 2]);
    M2 = fmaxf(M2, a.ws_ml[(rec0 + 2 * s + 1) * 2]);
  }
  float L1 = 0.f, L2 = 0.f, O1 = 0.f, O2 = 0.f;
  for (int s = 0; s < S && r_ok; ++s) {
    const size_t r1 = rec0 + 2 * s, r2 = r1 + 1;
    const float ma = a.ws_ml[r1 * 2], mb = a.ws_ml[r2 * 2];
    // a split with no keys has m = -inf and l = 0; it contributes nothing
    const float f1 = ma == -INFINITY ? 0.f : ex2(ma - M1);
    const float f2 = mb == -INFINITY ? 0.f : ex2(mb - M2);
    L1 = fmaf(f1, a.ws_ml[r1 * 2 + 1], L1);
    L2 = fmaf(f2, a.ws_ml[r2 * 2 + 1], L2);
    O1 = fmaf(f1, a.ws_o[r1 * DV + c], O1);
    O2 = fmaf(f2, a.ws_o[r2 * DV + c], O2);
  }
  const float lam = a.lambda[h];
  // no visible key (kv_len = 0): both sums are 0 and the output is 0
  float y = (L1 > 0.f ? O1 / L1 : 0.f) - lam * (L2 > 0.f ? O2 / L2 : 0.f);
  if (a.apply_norm) {
    const float ss = warp_sum(y * y);
    if ((c & 31) == 0) red[c >> 5] = ss;
    __syncthreads();
    const float tot = (red[0] + red[1]) + (red[2] + red[3]);
    y = y * rsqrtf(tot * (1.f / DV) + a.eps) * (1.f - a.lambda_init[0]);
  }
  const int64_t o_off = b * a.os[0] + (int64_t)h * a.os[1];
  if (in_bounds(o_off + c, 1, a.ext_out, a.dev_status, a.dbg_status))
    static_cast<__nv_bfloat16*>(a.out)[o_off + c] = __float2bfloat16_rn(y);
}

int decode_v1_default_splits(int B, int L, int H) {
  const int units = B * H;
  int s = (L + 8191) / 8192;
  const int min_blocks = 2 * 148 * 2;
  if (units > 0 && units * s < min_blocks) s = (min_blocks + units - 1) / units;
  const int max_s = (L + CH - 1) / CH;
  if (s > max_s) s = max_s;
  return s < 1 ? 1 : s;
}

cudaError_t launch_decode_v1(const DecodeArgs& a, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(decode_v1_split_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_v1_split_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  if (a.block_table)
    decode_v1_split_kernel<true><<<dim3(a.splits, a.Hq, a.B), THREADS, SMEM_BYTES, stream>>>(a);
  else
    decode_v1_split_kernel<false><<<dim3(a.splits, a.Hq, a.B), THREADS, SMEM_BYTES, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_v1_combine_kernel<<<dim3(a.Hq, a.B), DV, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace diffattn
