// backward.cu -- gradients of the differential attention prefill (SIMT, fp32 arithmetic).
//
// The pages present lambda and the projections as learnable and the layer as pre-trained
// ("Differential Attention (V2)", Key Terms, "lambda"; "V1 vs V2"), so training needs the
// gradient of the forward operator
//   A_b = softmax(Q_b K_b^T / sqrt(d)),  O = A_1 V - lambda A_2 V,
//   V1: y = (1 - lambda_init) O / sqrt(mean O^2 + eps);  V2: y = O.
// Given dy it is, per row i (softmax backward with delta_b,i = sum_j A_b,ij dA_b,ij):
//   dO      = V1: s/r (dy - O (dy . O)/(n r^2)) ; V2: dy
//   dp_ij   = dO_i . v_j,  delta_1 = dO_i . O_1,i,  delta_2 = dO_i . O_2,i
//   dS_1,ij = A_1,ij (dp_ij - delta_1),  dS_2,ij = -lambda A_2,ij (dp_ij - delta_2)
//   dQ_b    = dS_b K_b / sqrt(d),  dK_b = dS_b^T Q_b / sqrt(d),  dV = (A_1 - lambda A_2)^T dO
//   dlambda = -sum_i dO_i . O_2,i
// with O_b = A_b V (delta_1 uses sum_j A_1,ij dp_ij = dO_i . O_1,i; delta_2 carries the -lambda
// of dA_2 inside dS_2).
//
// Three launches, none with atomics (deterministic):
//   bwd_rows_kernel : one warp per (query row, unit), 8 rows per block sharing staged key
//                     rows (see below). Sweep 1 recomputes both branches'
//                     softmax statistics and O_1, O_2; it forms dO (the V1 norm backward),
//                     delta_1, delta_2, the row's dlambda share, and stores them with the
//                     log-sum-exps. Sweep 2 recomputes A_b row by row and accumulates dQ.
//   bwd_keys_kernel : one warp per (key row, KV head), 8 rows per block sharing staged
//                     query rows: walks every query that sees the key,
//                     for every unit that reads this KV head (V2: the pairs of the GQA
//                     group, both branches), recomputing A_b from the stored log-sum-exps,
//                     and accumulates dK and dV.
//   bwd_dlambda_kernel : sums the per-row dlambda shares in a fixed order.
#include "common.cuh"
#include "kernels.h"

namespace diffattn {

namespace {
constexpr int kMaxD = 128;          // branch width
constexpr int kMaxDv = 2 * kMaxD;   // value width (V1: 2d)
constexpr int kPerLane = kMaxDv / 32;
constexpr int kPerLaneD = kMaxD / 32;

template <typename T>
__device__ __forceinline__ float4 ld4(const T* p);
template <>
__device__ __forceinline__ float4 ld4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 ld4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                     __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
}
__device__ __forceinline__ float ld1(const float* p) { return *p; }
__device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// dot product of a global row (T) and a shared fp32 row, n a multiple of 4
template <typename T>
__device__ __forceinline__ float dot_row(const T* g, const float* s, int n) {
  float acc = 0.f;
  for (int c = 0; c < n; c += 4) {
    const float4 x = ld4(g + c);
    const float4 y = *reinterpret_cast<const float4*>(s + c);
    acc = fmaf(x.x, y.x, acc);
    acc = fmaf(x.y, y.y, acc);
    acc = fmaf(x.z, y.z, acc);
    acc = fmaf(x.w, y.w, acc);
  }
  return acc;
}

// visible keys of query row i: lo .. hi
__device__ __forceinline__ void key_range(const PrefillArgs& a, int i, int& lo, int& hi) {
  hi = a.causal ? i + (a.Nk - a.N) : a.Nk - 1;
  lo = (a.causal && a.window > 0) ? max(0, hi - a.window + 1) : 0;
}

// element offsets of unit u's branch rows (V1: head u, branch 2 at +d; V2: heads 2u, 2u+1
// and their shared KV head)
struct UnitRows {
  int64_t q1, q2, k1, k2, v;
};
__device__ __forceinline__ UnitRows unit_rows(const PrefillArgs& a, int u) {
  UnitRows r;
  if (a.variant == DIFFATTN_V1) {
    r.q1 = (int64_t)u * a.qs[2];
    r.q2 = r.q1 + a.d;
    r.k1 = (int64_t)u * a.ks[2];
    r.k2 = r.k1 + a.d;
    r.v = (int64_t)u * a.vs[2];
  } else {
    const int g = (2 * u) / a.group;
    r.q1 = (int64_t)(2 * u) * a.qs[2];
    r.q2 = (int64_t)(2 * u + 1) * a.qs[2];
    r.k1 = r.k2 = (int64_t)g * a.ks[2];
    r.v = (int64_t)g * a.vs[2];
  }
  return r;
}
}  // namespace

// Both passes run kRowWarps rows per block, one per warp, over the same unit (row pass) or
// KV head (key pass). Consecutive rows see nearly the same range of the other side, so the
// block walks the union of its rows' ranges in blocks of 32 rows of the other side: all
// warps stage those rows into shared memory as fp32 (one contiguous row per warp
// instruction), then every warp reads them from there (row r at stride width + 4 floats, so
// a quarter-warp reading 16 bytes from 8 different rows covers the 32 banks once). Warps
// whose own row is out of range still stage and meet every block barrier.
namespace {
constexpr int kRowWarps = 8;
constexpr int kBlk = 32;

// dot product of two 16-byte-aligned shared fp32 rows, n a multiple of 4, in the order of
// dot_row
__device__ __forceinline__ float dot_sm(const float* x, const float* y, int n) {
  float acc = 0.f;
  for (int c = 0; c < n; c += 4) {
    const float4 p = *reinterpret_cast<const float4*>(x + c);
    const float4 q = *reinterpret_cast<const float4*>(y + c);
    acc = fmaf(p.x, q.x, acc);
    acc = fmaf(p.y, q.y, acc);
    acc = fmaf(p.z, q.z, acc);
    acc = fmaf(p.w, q.w, acc);
  }
  return acc;
}

// rows r0 .. r0 + n - 1 of a global tensor (row stride rs elements, first column at col0)
// into shared rows of `width` floats at stride width + 4, by the block's warps
template <typename T>
__device__ __forceinline__ void stage_rows(float* dst, const T* src, int64_t rs, int64_t col0,
                                           int r0, int n, int width) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < n; r += kRowWarps) {
    const T* s = src + (int64_t)(r0 + r) * rs + col0;
    float* t = dst + r * (width + 4);
    for (int c = 4 * lane; c < width; c += 128) *reinterpret_cast<float4*>(t + c) = ld4(s + c);
  }
}

size_t bwd_simt_smem_bytes(int d, int dv) {
  const size_t stage = (size_t)kBlk * (2 * (d + 4) + (dv + 4)) + 4 * kBlk;
  return (stage + (size_t)kRowWarps * (2 * d + dv)) * sizeof(float);
}
}  // namespace

template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32) bwd_rows_kernel(BwdArgs g) {
  const PrefillArgs& a = g.f;
  const int d = a.d, dv = a.dv;
  extern __shared__ __align__(16) float sm[];
  float* k1s = sm;                          // [kBlk][d + 1]
  float* k2s = k1s + kBlk * (d + 4);        // [kBlk][d + 1]
  float* vsb = k2s + kBlk * (d + 4);        // [kBlk][dv + 1]
  float* qsm = vsb + kBlk * (dv + 4) + 4 * kBlk;  // [warp][2][d]
  float* dsm = qsm + kRowWarps * 2 * d;     // [warp][dv]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ib = blockIdx.x * kRowWarps;
  const int i = ib + warp;
  const int u = blockIdx.y, b = blockIdx.z;
  const T* k = static_cast<const T*>(a.k) + b * a.ks[0];
  const T* v = static_cast<const T*>(a.v) + b * a.vs[0];
  const UnitRows ur = unit_rows(a, u);
  bool valid = i < a.N;
  int lo = 0, hi = -1;
  if (valid) key_range(a, i, lo, hi);
  // the block's key range: key_range is monotone in the query row
  int blo, bhi, t0, t1;
  key_range(a, ib, blo, t0);
  key_range(a, min(ib + kRowWarps, a.N) - 1, t1, bhi);
  const int64_t row = ((int64_t)b * a.N + (valid ? i : 0)) * a.units + u;
  if (valid) {
    // (bounds-checked build) every row this warp reads or writes
    const int64_t qo = b * a.qs[0] + (int64_t)i * a.qs[1];
    const int64_t dq_off = a.variant == DIFFATTN_V1 ? (((int64_t)b * a.N + i) * a.units + u) * 2 * d
                                                    : (((int64_t)b * a.N + i) * a.Hq + 2 * u) * d;
    valid = in_bounds(qo + ur.q1, d, a.ext_q, a.dev_status, a.dbg_status) &&
            in_bounds(qo + ur.q2, d, a.ext_q, a.dev_status, a.dbg_status) &&
            in_bounds(b * g.dys[0] + (int64_t)i * g.dys[1] + u * g.dys[2], dv, a.ext_out,
                      a.dev_status, a.dbg_status) &&
            in_bounds((g.w_do - g.w_base) + row * dv, dv, g.ext_ws, a.dev_status, a.dbg_status) &&
            in_bounds((g.w_st - g.w_base) + row * 4, 4, g.ext_ws, a.dev_status, a.dbg_status) &&
            in_bounds((g.w_dl - g.w_base) + ((int64_t)b * a.units + u) * a.N + i, 1, g.ext_ws,
                      a.dev_status, a.dbg_status) &&
            in_bounds(dq_off, 2 * d, g.ext_dq, a.dev_status, a.dbg_status);
  }
  // (bounds-checked build) the block's first and last key rows bound the staged ones; the
  // strides are non-negative
  bool keys_ok = true;
  if (blo <= bhi)
    for (int e = 0; e < 2; ++e) {
      const int jj = e ? bhi : blo;
      keys_ok = keys_ok &&
                in_bounds(b * a.ks[0] + (int64_t)jj * a.ks[1] + ur.k1, d, a.ext_k, a.dev_status, a.dbg_status) &&
                in_bounds(b * a.ks[0] + (int64_t)jj * a.ks[1] + ur.k2, d, a.ext_k, a.dev_status, a.dbg_status) &&
                in_bounds(b * a.vs[0] + (int64_t)jj * a.vs[1] + ur.v, dv, a.ext_v, a.dev_status, a.dbg_status);
    }
  if (!keys_ok) bhi = blo - 1;  // uniform over the block: stage nothing
  valid = valid && keys_ok;
  float* qw = qsm + warp * 2 * d;
  float* dw = dsm + warp * dv;
  if (valid) {
    const T* q = static_cast<const T*>(a.q) + b * a.qs[0] + (int64_t)i * a.qs[1];
    for (int c = lane; c < d; c += 32) {
      qw[c] = ld1(q + ur.q1 + c);
      qw[d + c] = ld1(q + ur.q2 + c);
    }
  }
  __syncwarp();
  const float scale = 1.0f / sqrtf((float)d);
  const float lam = a.lambda[u];

  // ---- sweep 1: statistics and O_1, O_2 of both branches
  float m1 = -INFINITY, m2 = -INFINITY, l1 = 0.f, l2 = 0.f;
  float o1[kPerLane], o2[kPerLane];
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) o1[t] = o2[t] = 0.f;
  for (int j0 = blo; j0 <= bhi; j0 += kBlk) {
    const int jn = min(kBlk, bhi - j0 + 1);
    stage_rows(k1s, k, a.ks[1], ur.k1, j0, jn, d);
    stage_rows(k2s, k, a.ks[1], ur.k2, j0, jn, d);
    stage_rows(vsb, v, a.vs[1], ur.v, j0, jn, dv);
    __syncthreads();
    if (valid && j0 <= hi && j0 + jn - 1 >= lo) {
      const int j = j0 + lane;
      const bool vis = lane < jn && j >= lo && j <= hi;
      float s1 = -INFINITY, s2 = -INFINITY;
      if (vis) {
        s1 = dot_sm(k1s + lane * (d + 4), qw, d) * scale;
        s2 = dot_sm(k2s + lane * (d + 4), qw + d, d) * scale;
      }
      const float n1 = fmaxf(m1, warp_max(s1)), n2 = fmaxf(m2, warp_max(s2));
      const float al1 = (m1 == -INFINITY) ? 0.f : expf(m1 - n1);
      const float al2 = (m2 == -INFINITY) ? 0.f : expf(m2 - n2);
      const float p1 = vis ? expf(s1 - n1) : 0.f;
      const float p2 = vis ? expf(s2 - n2) : 0.f;
      l1 = l1 * al1 + warp_sum(p1);
      l2 = l2 * al2 + warp_sum(p2);
      m1 = n1;
      m2 = n2;
#pragma unroll
      for (int t = 0; t < kPerLane; ++t) {
        o1[t] *= al1;
        o2[t] *= al2;
      }
      for (int jj = 0; jj < jn; ++jj) {
        const float w1 = __shfl_sync(0xffffffffu, p1, jj);
        const float w2 = __shfl_sync(0xffffffffu, p2, jj);
        const float* vr = vsb + jj * (dv + 4);
#pragma unroll
        for (int t = 0; t < kPerLane; ++t) {
          const int c = lane + 32 * t;
          if (c < dv) {
            const float x = vr[c];
            o1[t] = fmaf(w1, x, o1[t]);
            o2[t] = fmaf(w2, x, o2[t]);
          }
        }
      }
    }
    __syncthreads();
  }

  // ---- dO (through the V1 norm), delta_1, delta_2, dlambda share
  float dO[kPerLane];
  float lse1 = 0.f, lse2 = 0.f, delta1 = 0.f, delta2 = 0.f;
  if (valid) {
    const T* dy = static_cast<const T*>(g.dy) + b * g.dys[0] + (int64_t)i * g.dys[1] + u * g.dys[2];
    float so = 0.f, sdy = 0.f;
#pragma unroll
    for (int t = 0; t < kPerLane; ++t) {
      const int c = lane + 32 * t;
      o1[t] /= l1;
      o2[t] /= l2;
      const float o = o1[t] - lam * o2[t];
      dO[t] = (c < dv) ? ld1(dy + c) : 0.f;
      if (c < dv) {
        so = fmaf(o, o, so);
        sdy = fmaf(dO[t], o, sdy);
      }
    }
    if (a.apply_norm) {
      so = warp_sum(so);
      sdy = warp_sum(sdy);
      const float r2 = so / (float)dv + a.eps;
      const float r = sqrtf(r2);
      const float s = 1.0f - a.lambda_init[0];
      const float proj = sdy / ((float)dv * r2);
#pragma unroll
      for (int t = 0; t < kPerLane; ++t) {
        const float o = o1[t] - lam * o2[t];
        dO[t] = s / r * (dO[t] - o * proj);
      }
    }
    float e1 = 0.f, e2 = 0.f;
#pragma unroll
    for (int t = 0; t < kPerLane; ++t) {
      if (lane + 32 * t < dv) {
        e1 = fmaf(dO[t], o1[t], e1);
        e2 = fmaf(dO[t], o2[t], e2);
      }
    }
    delta1 = warp_sum(e1);
    delta2 = warp_sum(e2);
    float* wdo = g.w_do + row * dv;
#pragma unroll
    for (int t = 0; t < kPerLane; ++t) {
      const int c = lane + 32 * t;
      if (c < dv) {
        dw[c] = dO[t];
        wdo[c] = dO[t];
      }
    }
    lse1 = m1 + logf(l1);
    lse2 = m2 + logf(l2);
    if (lane == 0) {
      *reinterpret_cast<float4*>(g.w_st + row * 4) = make_float4(lse1, lse2, delta1, delta2);
      g.w_dl[((int64_t)b * a.units + u) * a.N + i] = -delta2;
    }
  }
  __syncwarp();

  // ---- sweep 2: dQ_b = sum_j dS_b,ij k_b,j / sqrt(d)
  float dq1[kPerLaneD], dq2[kPerLaneD];
#pragma unroll
  for (int t = 0; t < kPerLaneD; ++t) dq1[t] = dq2[t] = 0.f;
  for (int j0 = blo; j0 <= bhi; j0 += kBlk) {
    const int jn = min(kBlk, bhi - j0 + 1);
    stage_rows(k1s, k, a.ks[1], ur.k1, j0, jn, d);
    stage_rows(k2s, k, a.ks[1], ur.k2, j0, jn, d);
    stage_rows(vsb, v, a.vs[1], ur.v, j0, jn, dv);
    __syncthreads();
    if (valid && j0 <= hi && j0 + jn - 1 >= lo) {
      const int j = j0 + lane;
      float ds1 = 0.f, ds2 = 0.f;
      if (lane < jn && j >= lo && j <= hi) {
        const float s1 = dot_sm(k1s + lane * (d + 4), qw, d) * scale;
        const float s2 = dot_sm(k2s + lane * (d + 4), qw + d, d) * scale;
        const float dp = dot_sm(vsb + lane * (dv + 4), dw, dv);
        ds1 = expf(s1 - lse1) * (dp - delta1);
        ds2 = -lam * expf(s2 - lse2) * (dp - delta2);
      }
      for (int jj = 0; jj < jn; ++jj) {
        const float w1 = __shfl_sync(0xffffffffu, ds1, jj);
        const float w2 = __shfl_sync(0xffffffffu, ds2, jj);
        const float* r1 = k1s + jj * (d + 4);
        const float* r2 = k2s + jj * (d + 4);
#pragma unroll
        for (int t = 0; t < kPerLaneD; ++t) {
          const int c = lane + 32 * t;
          if (c < d) {
            dq1[t] = fmaf(w1, r1[c], dq1[t]);
            dq2[t] = fmaf(w2, r2[c], dq2[t]);
          }
        }
      }
    }
    __syncthreads();
  }
  if (!valid) return;
  // dq: dense fp32 in q's shape (V1 [B,N,H,2,d]; V2 [B,N,Hq,d])
  float* dq_1;
  float* dq_2;
  if (a.variant == DIFFATTN_V1) {
    dq_1 = g.dq + (((int64_t)b * a.N + i) * a.units + u) * 2 * d;
    dq_2 = dq_1 + d;
  } else {
    dq_1 = g.dq + (((int64_t)b * a.N + i) * a.Hq + 2 * u) * d;
    dq_2 = dq_1 + d;
  }
#pragma unroll
  for (int t = 0; t < kPerLaneD; ++t) {
    const int c = lane + 32 * t;
    if (c < d) {
      dq_1[c] = dq1[t] * scale;
      dq_2[c] = dq2[t] * scale;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32) bwd_keys_kernel(BwdArgs g) {
  const PrefillArgs& a = g.f;
  const int d = a.d, dv = a.dv;
  extern __shared__ __align__(16) float sm[];
  float* q1s = sm;                          // [kBlk][d + 1]
  float* q2s = q1s + kBlk * (d + 4);        // [kBlk][d + 1]
  float* dos = q2s + kBlk * (d + 4);        // [kBlk][dv + 1]
  float4* sts = reinterpret_cast<float4*>(dos + kBlk * (dv + 4));  // [kBlk]
  float* ksm = reinterpret_cast<float*>(sts + kBlk);  // [warp][2][d]
  float* vsm = ksm + kRowWarps * 2 * d;     // [warp][dv]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jb = blockIdx.x * kRowWarps;
  const int j = jb + warp;                  // key row
  const int kh = blockIdx.y;                // V1 head / V2 KV head
  const int b = blockIdx.z;
  const bool v1 = a.variant == DIFFATTN_V1;
  bool valid = j < a.Nk;
  const int64_t k_off = b * a.ks[0] + (int64_t)(valid ? j : 0) * a.ks[1] + (int64_t)kh * a.ks[2];
  const int64_t v_off = b * a.vs[0] + (int64_t)(valid ? j : 0) * a.vs[1] + (int64_t)kh * a.vs[2];
  const int nkh = v1 ? a.units : a.Hkv;
  const int64_t krow = ((int64_t)b * a.Nk + (valid ? j : 0)) * nkh + kh;
  // (bounds-checked build) this key's rows and outputs
  if (valid)
    valid = in_bounds(k_off, v1 ? 2 * d : d, a.ext_k, a.dev_status, a.dbg_status) &&
            in_bounds(v_off, dv, a.ext_v, a.dev_status, a.dbg_status) &&
            in_bounds(krow * (v1 ? 2 * d : d), v1 ? 2 * d : d, g.ext_dk, a.dev_status, a.dbg_status) &&
            in_bounds(krow * dv, dv, g.ext_dv, a.dev_status, a.dbg_status);
  float* kw = ksm + warp * 2 * d;
  float* vw = vsm + warp * dv;
  if (valid) {
    const T* kr = static_cast<const T*>(a.k) + k_off;
    const T* vr = static_cast<const T*>(a.v) + v_off;
    for (int c = lane; c < d; c += 32) {
      kw[c] = ld1(kr + c);
      kw[d + c] = ld1(kr + (v1 ? d : 0) + c);
    }
    for (int c = lane; c < dv; c += 32) vw[c] = ld1(vr + c);
  }
  __syncwarp();
  const float scale = 1.0f / sqrtf((float)d);
  // queries that see key j: i + off >= j (causal) and i + off - window < j (window); both
  // ends are monotone in j, so the block's range is the first key's start to the last's end
  const int off = a.Nk - a.N;
  auto query_range = [&](int jj, int& lo, int& hi) {
    lo = 0;
    hi = a.N - 1;
    if (a.causal) {
      lo = max(0, jj - off);
      if (a.window > 0) hi = min(a.N - 1, jj - off + a.window - 1);
    }
  };
  int i_lo = 0, i_hi = -1, bilo, bihi, t0, t1;
  if (valid) query_range(j, i_lo, i_hi);
  query_range(jb, bilo, t0);
  query_range(min(jb + kRowWarps, a.Nk) - 1, t1, bihi);
  // units reading this KV head: V1 the head itself; V2 the pairs of its GQA group
  const int u_lo = v1 ? kh : kh * (a.group / 2);
  const int u_hi = v1 ? kh + 1 : (kh + 1) * (a.group / 2);

  float dk1[kPerLaneD], dk2[kPerLaneD], dvv[kPerLane];
#pragma unroll
  for (int t = 0; t < kPerLaneD; ++t) dk1[t] = dk2[t] = 0.f;
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) dvv[t] = 0.f;

  for (int u = u_lo; u < u_hi; ++u) {
    const float lam = a.lambda[u];
    const UnitRows ur = unit_rows(a, u);
    const T* q = static_cast<const T*>(a.q) + b * a.qs[0];
    const float* wdo = g.w_do + ((int64_t)b * a.N) * a.units * dv;
    const float* wst = g.w_st + ((int64_t)b * a.N) * a.units * 4;
    int hi_u = bihi;
    if (bilo <= bihi) {
      // (bounds-checked build) the first and last query rows bound the staged ones
      bool ok = true;
      for (int e = 0; e < 2; ++e) {
        const int ii = e ? bihi : bilo;
        const int64_t row = ((int64_t)b * a.N + ii) * a.units + u;
        ok = ok && in_bounds(b * a.qs[0] + (int64_t)ii * a.qs[1] + ur.q1, d, a.ext_q, a.dev_status, a.dbg_status) &&
             in_bounds(b * a.qs[0] + (int64_t)ii * a.qs[1] + ur.q2, d, a.ext_q, a.dev_status, a.dbg_status) &&
             in_bounds((g.w_st - g.w_base) + row * 4, 4, g.ext_ws, a.dev_status, a.dbg_status) &&
             in_bounds((g.w_do - g.w_base) + row * dv, dv, g.ext_ws, a.dev_status, a.dbg_status);
      }
      if (!ok) {
        hi_u = bilo - 1;  // uniform over the block: stage nothing for this unit
        valid = false;
      }
    }
    for (int i0 = bilo; i0 <= hi_u; i0 += kBlk) {
      const int in = min(kBlk, hi_u - i0 + 1);
      stage_rows(q1s, q, a.qs[1], ur.q1, i0, in, d);
      stage_rows(q2s, q, a.qs[1], ur.q2, i0, in, d);
      stage_rows(dos, wdo, (int64_t)a.units * dv, (int64_t)u * dv, i0, in, dv);
      if (threadIdx.x < in)
        sts[threadIdx.x] = *reinterpret_cast<const float4*>(wst + ((int64_t)(i0 + threadIdx.x) * a.units + u) * 4);
      __syncthreads();
      if (valid && i0 <= i_hi && i0 + in - 1 >= i_lo) {
        const int i = i0 + lane;
        float pv = 0.f, ds1 = 0.f, ds2 = 0.f;
        if (lane < in && i >= i_lo && i <= i_hi) {
          const float4 st = sts[lane];
          const float s1 = dot_sm(q1s + lane * (d + 4), kw, d) * scale;
          const float s2 = dot_sm(q2s + lane * (d + 4), kw + d, d) * scale;
          const float p1 = expf(s1 - st.x), p2 = expf(s2 - st.y);
          const float dp = dot_sm(dos + lane * (dv + 4), vw, dv);
          pv = p1 - lam * p2;
          ds1 = p1 * (dp - st.z);
          ds2 = -lam * p2 * (dp - st.w);
        }
        for (int ii = 0; ii < in; ++ii) {
          const float w = __shfl_sync(0xffffffffu, pv, ii);
          const float w1 = __shfl_sync(0xffffffffu, ds1, ii);
          const float w2 = __shfl_sync(0xffffffffu, ds2, ii);
          const float* dor = dos + ii * (dv + 4);
          const float* r1 = q1s + ii * (d + 4);
          const float* r2 = q2s + ii * (d + 4);
#pragma unroll
          for (int t = 0; t < kPerLane; ++t) {
            const int c = lane + 32 * t;
            if (c < dv) dvv[t] = fmaf(w, dor[c], dvv[t]);
          }
#pragma unroll
          for (int t = 0; t < kPerLaneD; ++t) {
            const int c = lane + 32 * t;
            if (c < d) {
              dk1[t] = fmaf(w1, r1[c], dk1[t]);
              dk2[t] = fmaf(w2, r2[c], dk2[t]);
            }
          }
        }
      }
      __syncthreads();
    }
  }
  if (!valid) return;
  // dense fp32 outputs in k's and v's shapes (V1 k [B,Nk,H,2,d], v [B,Nk,H,2d];
  // V2 k, v [B,Nk,Hkv,d]); V2's two branches read the same K row, so their parts add
#pragma unroll
  for (int t = 0; t < kPerLaneD; ++t) {
    const int c = lane + 32 * t;
    if (c < d) {
      if (v1) {
        g.dk[krow * 2 * d + c] = dk1[t] * scale;
        g.dk[krow * 2 * d + d + c] = dk2[t] * scale;
      } else {
        g.dk[krow * d + c] = (dk1[t] + dk2[t]) * scale;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    const int c = lane + 32 * t;
    if (c < dv) g.dv[krow * dv + c] = dvv[t];
  }
}

// dlambda[u] = sum over batch entries and rows of the per-row shares, in a fixed order
__global__ void __launch_bounds__(256) bwd_dlambda_kernel(BwdArgs g) {
  const PrefillArgs& a = g.f;
  __shared__ float red[256];
  const int u = blockIdx.x;
  float s = 0.f;
  for (int b = 0; b < a.B; ++b) {
    const float* w = g.w_dl + ((int64_t)b * a.units + u) * a.N;
    if (!in_bounds(w - g.w_base, a.N, g.ext_ws, a.dev_status, a.dbg_status)) continue;
    for (int i = threadIdx.x; i < a.N; i += 256) s += w[i];
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) g.dlambda[u] = red[0];
}

size_t bwd_workspace_bytes(int B, int N, int units, int dv) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t rows = (size_t)B * N * units;
  return up(rows * dv * sizeof(float)) + up(rows * 4 * sizeof(float)) + up(rows * sizeof(float));
}

cudaError_t launch_backward(BwdArgs g, void* workspace, cudaStream_t stream) {
  const PrefillArgs& a = g.f;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t rows = (size_t)a.B * a.N * a.units;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  g.w_do = reinterpret_cast<float*>(w);
  g.w_st = reinterpret_cast<float*>(w + up(rows * a.dv * sizeof(float)));
  g.w_dl = reinterpret_cast<float*>(w + up(rows * a.dv * sizeof(float)) + up(rows * 4 * sizeof(float)));
  g.w_base = g.w_do;
  const dim3 grid_rows((a.N + kRowWarps - 1) / kRowWarps, a.units, a.B);
  const int nkh = a.variant == DIFFATTN_V1 ? a.units : a.Hkv;
  const dim3 grid_keys((a.Nk + kRowWarps - 1) / kRowWarps, nkh, a.B);
  const size_t smem = bwd_simt_smem_bytes(a.d, a.dv);
  // (d <= 128, dv <= 256: at most 85 KB, above the 48 KB default)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    const int max_smem = (int)bwd_simt_smem_bytes(kMaxD, kMaxDv);
    const void* fns[4] = {(const void*)bwd_rows_kernel<__nv_bfloat16>, (const void*)bwd_keys_kernel<__nv_bfloat16>,
                          (const void*)bwd_rows_kernel<float>, (const void*)bwd_keys_kernel<float>};
    for (const void* fn : fns) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
      if (e != cudaSuccess) return e;
    }
    if (dev < 64) attr_set[dev] = true;
  }
  if (g.bf16) {
    bwd_rows_kernel<__nv_bfloat16><<<grid_rows, kRowWarps * 32, smem, stream>>>(g);
    bwd_keys_kernel<__nv_bfloat16><<<grid_keys, kRowWarps * 32, smem, stream>>>(g);
  } else {
    bwd_rows_kernel<float><<<grid_rows, kRowWarps * 32, smem, stream>>>(g);
    bwd_keys_kernel<float><<<grid_keys, kRowWarps * 32, smem, stream>>>(g);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_dlambda_reduce(g, stream);
}

cudaError_t launch_dlambda_reduce(const BwdArgs& g, cudaStream_t stream) {
  bwd_dlambda_kernel<<<g.f.units, 256, 0, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace diffattn
