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
//   bwd_rows_kernel : one warp per (query row, unit). Sweep 1 recomputes both branches'
//                     softmax statistics and O_1, O_2; it forms dO (the V1 norm backward),
//                     delta_1, delta_2, the row's dlambda share, and stores them with the
//                     log-sum-exps. Sweep 2 recomputes A_b row by row and accumulates dQ.
//   bwd_keys_kernel : one warp per (key row, KV head): walks every query that sees the key,
//                     for every unit that reads this KV head (V2: the pairs of the GQA
//                     group, both branches), recomputing A_b from the stored log-sum-exps,
//                     and accumulates dK and dV.
//   bwd_dlambda_kernel : sums the per-row dlambda shares in a fixed order.
#include "common.cuh"
#include "kernels.h"

namespace diffattn {

namespace {
constexpr int kWarps = 4;
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

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) bwd_rows_kernel(BwdArgs g) {
  const PrefillArgs& a = g.f;
  __shared__ __align__(16) float qsm[kWarps][2][kMaxD];
  __shared__ __align__(16) float dsm[kWarps][kMaxDv];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kWarps + warp;
  const int u = blockIdx.y, b = blockIdx.z;
  if (i >= a.N) return;
  const int d = a.d, dv = a.dv;
  const T* q = static_cast<const T*>(a.q) + b * a.qs[0] + (int64_t)i * a.qs[1];
  const T* k = static_cast<const T*>(a.k) + b * a.ks[0];
  const T* v = static_cast<const T*>(a.v) + b * a.vs[0];
  const UnitRows ur = unit_rows(a, u);
  int lo, hi;
  key_range(a, i, lo, hi);
  {
    // (bounds-checked build) every row this warp reads or writes; the strides are
    // non-negative, so the first and last key rows bound all the others
    const int64_t qo = b * a.qs[0] + (int64_t)i * a.qs[1];
    const int64_t row = ((int64_t)b * a.N + i) * a.units + u;
    const int64_t dq_off = a.variant == DIFFATTN_V1 ? (((int64_t)b * a.N + i) * a.units + u) * 2 * d
                                                    : (((int64_t)b * a.N + i) * a.Hq + 2 * u) * d;
    bool ok = in_bounds(qo + ur.q1, d, a.ext_q, a.dev_status, a.dbg_status) &&
              in_bounds(qo + ur.q2, d, a.ext_q, a.dev_status, a.dbg_status) &&
              in_bounds(b * g.dys[0] + (int64_t)i * g.dys[1] + u * g.dys[2], dv, a.ext_out,
                        a.dev_status, a.dbg_status) &&
              in_bounds((g.w_do - g.w_base) + row * dv, dv, g.ext_ws, a.dev_status, a.dbg_status) &&
              in_bounds((g.w_st - g.w_base) + row * 4, 4, g.ext_ws, a.dev_status, a.dbg_status) &&
              in_bounds((g.w_dl - g.w_base) + ((int64_t)b * a.units + u) * a.N + i, 1, g.ext_ws,
                        a.dev_status, a.dbg_status) &&
              in_bounds(dq_off, 2 * d, g.ext_dq, a.dev_status, a.dbg_status);
    if (lo <= hi)
      for (int e = 0; e < 2; ++e) {
        const int jj = e ? hi : lo;
        ok = ok && in_bounds(b * a.ks[0] + (int64_t)jj * a.ks[1] + ur.k1, d, a.ext_k, a.dev_status, a.dbg_status) &&
             in_bounds(b * a.ks[0] + (int64_t)jj * a.ks[1] + ur.k2, d, a.ext_k, a.dev_status, a.dbg_status) &&
             in_bounds(b * a.vs[0] + (int64_t)jj * a.vs[1] + ur.v, dv, a.ext_v, a.dev_status, a.dbg_status);
      }
    if (!ok) return;
  }
  for (int c = lane; c < d; c += 32) {
    qsm[warp][0][c] = ld1(q + ur.q1 + c);
    qsm[warp][1][c] = ld1(q + ur.q2 + c);
  }
  __syncwarp();
  const float scale = 1.0f / sqrtf((float)d);
  const float lam = a.lambda[u];

  // ---- sweep 1: statistics and O_1, O_2 of both branches
  float m1 = -INFINITY, m2 = -INFINITY, l1 = 0.f, l2 = 0.f;
  float o1[kPerLane], o2[kPerLane];
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) o1[t] = o2[t] = 0.f;
  for (int j0 = lo; j0 <= hi; j0 += 32) {
    const int j = j0 + lane;
    float s1 = -INFINITY, s2 = -INFINITY;
    if (j <= hi) {
      s1 = dot_row(k + (int64_t)j * a.ks[1] + ur.k1, qsm[warp][0], d) * scale;
      s2 = dot_row(k + (int64_t)j * a.ks[1] + ur.k2, qsm[warp][1], d) * scale;
    }
    const float n1 = fmaxf(m1, warp_max(s1)), n2 = fmaxf(m2, warp_max(s2));
    const float al1 = (m1 == -INFINITY) ? 0.f : expf(m1 - n1);
    const float al2 = (m2 == -INFINITY) ? 0.f : expf(m2 - n2);
    const float p1 = (j <= hi) ? expf(s1 - n1) : 0.f;
    const float p2 = (j <= hi) ? expf(s2 - n2) : 0.f;
    l1 = l1 * al1 + warp_sum(p1);
    l2 = l2 * al2 + warp_sum(p2);
    m1 = n1;
    m2 = n2;
#pragma unroll
    for (int t = 0; t < kPerLane; ++t) {
      o1[t] *= al1;
      o2[t] *= al2;
    }
    const int jn = min(32, hi - j0 + 1);
    for (int jj = 0; jj < jn; ++jj) {
      const float w1 = __shfl_sync(0xffffffffu, p1, jj);
      const float w2 = __shfl_sync(0xffffffffu, p2, jj);
      const T* vr = v + (int64_t)(j0 + jj) * a.vs[1] + ur.v;
#pragma unroll
      for (int t = 0; t < kPerLane; ++t) {
        const int c = lane + 32 * t;
        if (c < dv) {
          const float x = ld1(vr + c);
          o1[t] = fmaf(w1, x, o1[t]);
          o2[t] = fmaf(w2, x, o2[t]);
        }
      }
    }
  }

  // ---- dO (through the V1 norm), delta_1, delta_2, dlambda share
  const T* dy = static_cast<const T*>(g.dy) + b * g.dys[0] + (int64_t)i * g.dys[1] + u * g.dys[2];
  float dO[kPerLane];
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
  const float delta1 = warp_sum(e1), delta2 = warp_sum(e2);
  const int64_t row = ((int64_t)b * a.N + i) * a.units + u;
  float* wdo = g.w_do + row * dv;
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    const int c = lane + 32 * t;
    if (c < dv) {
      dsm[warp][c] = dO[t];
      wdo[c] = dO[t];
    }
  }
  const float lse1 = m1 + logf(l1), lse2 = m2 + logf(l2);
  if (lane == 0) {
    float4 st = make_float4(lse1, lse2, delta1, delta2);
    *reinterpret_cast<float4*>(g.w_st + row * 4) = st;
    g.w_dl[((int64_t)b * a.units + u) * a.N + i] = -delta2;
  }
  __syncwarp();

  // ---- sweep 2: dQ_b = sum_j dS_b,ij k_b,j / sqrt(d)
  float dq1[kPerLaneD], dq2[kPerLaneD];
#pragma unroll
  for (int t = 0; t < kPerLaneD; ++t) dq1[t] = dq2[t] = 0.f;
  for (int j0 = lo; j0 <= hi; j0 += 32) {
    const int j = j0 + lane;
    float ds1 = 0.f, ds2 = 0.f;
    if (j <= hi) {
      const float s1 = dot_row(k + (int64_t)j * a.ks[1] + ur.k1, qsm[warp][0], d) * scale;
      const float s2 = dot_row(k + (int64_t)j * a.ks[1] + ur.k2, qsm[warp][1], d) * scale;
      const float dp = dot_row(v + (int64_t)j * a.vs[1] + ur.v, dsm[warp], dv);
      ds1 = expf(s1 - lse1) * (dp - delta1);
      ds2 = -lam * expf(s2 - lse2) * (dp - delta2);
    }
    const int jn = min(32, hi - j0 + 1);
    for (int jj = 0; jj < jn; ++jj) {
      const float w1 = __shfl_sync(0xffffffffu, ds1, jj);
      const float w2 = __shfl_sync(0xffffffffu, ds2, jj);
      const T* kr = k + (int64_t)(j0 + jj) * a.ks[1];
#pragma unroll
      for (int t = 0; t < kPerLaneD; ++t) {
        const int c = lane + 32 * t;
        if (c < d) {
          dq1[t] = fmaf(w1, ld1(kr + ur.k1 + c), dq1[t]);
          dq2[t] = fmaf(w2, ld1(kr + ur.k2 + c), dq2[t]);
        }
      }
    }
  }
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
__global__ void __launch_bounds__(kWarps * 32) bwd_keys_kernel(BwdArgs g) {
  const PrefillArgs& a = g.f;
  __shared__ __align__(16) float ksm[kWarps][2][kMaxD];
  __shared__ __align__(16) float vsm[kWarps][kMaxDv];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kWarps + warp;  // key row
  const int kh = blockIdx.y;                 // V1 head / V2 KV head
  const int b = blockIdx.z;
  if (j >= a.Nk) return;
  const int d = a.d, dv = a.dv;
  const bool v1 = a.variant == DIFFATTN_V1;
  const int64_t k_off = b * a.ks[0] + (int64_t)j * a.ks[1] + (int64_t)kh * a.ks[2];
  const int64_t v_off = b * a.vs[0] + (int64_t)j * a.vs[1] + (int64_t)kh * a.vs[2];
  const int nkh_ = v1 ? a.units : a.Hkv;
  const int64_t krow_ = ((int64_t)b * a.Nk + j) * nkh_ + kh;
  // (bounds-checked build) this key's rows and outputs
  if (!(in_bounds(k_off, v1 ? 2 * d : d, a.ext_k, a.dev_status, a.dbg_status) &&
        in_bounds(v_off, dv, a.ext_v, a.dev_status, a.dbg_status) &&
        in_bounds(krow_ * (v1 ? 2 * d : d), v1 ? 2 * d : d, g.ext_dk, a.dev_status, a.dbg_status) &&
        in_bounds(krow_ * dv, dv, g.ext_dv, a.dev_status, a.dbg_status)))
    return;
  const T* kr = static_cast<const T*>(a.k) + k_off;
  const T* vr = static_cast<const T*>(a.v) + v_off;
  for (int c = lane; c < d; c += 32) {
    ksm[warp][0][c] = ld1(kr + c);
    ksm[warp][1][c] = ld1(kr + (v1 ? d : 0) + c);
  }
  for (int c = lane; c < dv; c += 32) vsm[warp][c] = ld1(vr + c);
  __syncwarp();
  const float scale = 1.0f / sqrtf((float)d);
  // queries that see key j: i + off >= j (causal) and i + off - window < j (window)
  const int off = a.Nk - a.N;
  int i_lo = 0, i_hi = a.N - 1;
  if (a.causal) {
    i_lo = max(0, j - off);
    if (a.window > 0) i_hi = min(a.N - 1, j - off + a.window - 1);
  }
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
    if (i_lo <= i_hi) {
      // (bounds-checked build) the first and last query rows bound the ones in between
      bool ok = true;
      for (int e = 0; e < 2; ++e) {
        const int ii = e ? i_hi : i_lo;
        const int64_t row = ((int64_t)b * a.N + ii) * a.units + u;
        ok = ok && in_bounds(b * a.qs[0] + (int64_t)ii * a.qs[1] + ur.q1, d, a.ext_q, a.dev_status, a.dbg_status) &&
             in_bounds(b * a.qs[0] + (int64_t)ii * a.qs[1] + ur.q2, d, a.ext_q, a.dev_status, a.dbg_status) &&
             in_bounds((g.w_st - g.w_base) + row * 4, 4, g.ext_ws, a.dev_status, a.dbg_status) &&
             in_bounds((g.w_do - g.w_base) + row * dv, dv, g.ext_ws, a.dev_status, a.dbg_status);
      }
      if (!ok) return;
    }
    for (int i0 = i_lo; i0 <= i_hi; i0 += 32) {
      const int i = i0 + lane;
      float pv = 0.f, ds1 = 0.f, ds2 = 0.f;
      if (i <= i_hi) {
        const int64_t row = ((int64_t)b * a.N + i) * a.units + u;
        const float4 st = *reinterpret_cast<const float4*>(g.w_st + row * 4);
        const float s1 = dot_row(q + (int64_t)i * a.qs[1] + ur.q1, ksm[warp][0], d) * scale;
        const float s2 = dot_row(q + (int64_t)i * a.qs[1] + ur.q2, ksm[warp][1], d) * scale;
        const float p1 = expf(s1 - st.x), p2 = expf(s2 - st.y);
        const float dp = dot_row(g.w_do + row * dv, vsm[warp], dv);
        pv = p1 - lam * p2;
        ds1 = p1 * (dp - st.z);
        ds2 = -lam * p2 * (dp - st.w);
      }
      const int in = min(32, i_hi - i0 + 1);
      for (int ii = 0; ii < in; ++ii) {
        const float w = __shfl_sync(0xffffffffu, pv, ii);
        const float w1 = __shfl_sync(0xffffffffu, ds1, ii);
        const float w2 = __shfl_sync(0xffffffffu, ds2, ii);
        const int64_t row = ((int64_t)b * a.N + i0 + ii) * a.units + u;
        const float* dor = g.w_do + row * dv;
        const T* qr = q + (int64_t)(i0 + ii) * a.qs[1];
#pragma unroll
        for (int t = 0; t < kPerLane; ++t) {
          const int c = lane + 32 * t;
          if (c < dv) dvv[t] = fmaf(w, dor[c], dvv[t]);
        }
#pragma unroll
        for (int t = 0; t < kPerLaneD; ++t) {
          const int c = lane + 32 * t;
          if (c < d) {
            dk1[t] = fmaf(w1, ld1(qr + ur.q1 + c), dk1[t]);
            dk2[t] = fmaf(w2, ld1(qr + ur.q2 + c), dk2[t]);
          }
        }
      }
    }
  }
  // dense fp32 outputs in k's and v's shapes (V1 k [B,Nk,H,2,d], v [B,Nk,H,2d];
  // V2 k, v [B,Nk,Hkv,d]); V2's two branches read the same K row, so their parts add
  const int nkh = v1 ? a.units : a.Hkv;
  const int64_t krow = ((int64_t)b * a.Nk + j) * nkh + kh;
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
  const dim3 grid_rows((a.N + kWarps - 1) / kWarps, a.units, a.B);
  const int nkh = a.variant == DIFFATTN_V1 ? a.units : a.Hkv;
  const dim3 grid_keys((a.Nk + kWarps - 1) / kWarps, nkh, a.B);
  if (g.bf16) {
    bwd_rows_kernel<__nv_bfloat16><<<grid_rows, kWarps * 32, 0, stream>>>(g);
    bwd_keys_kernel<__nv_bfloat16><<<grid_keys, kWarps * 32, 0, stream>>>(g);
  } else {
    bwd_rows_kernel<float><<<grid_rows, kWarps * 32, 0, stream>>>(g);
    bwd_keys_kernel<float><<<grid_keys, kWarps * 32, 0, stream>>>(g);
  }
  return launch_dlambda_reduce(g, stream);
}

cudaError_t launch_dlambda_reduce(const BwdArgs& g, cudaStream_t stream) {
  bwd_dlambda_kernel<<<g.f.units, 256, 0, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace diffattn
