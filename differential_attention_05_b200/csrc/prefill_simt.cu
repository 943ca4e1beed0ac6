// prefill_simt.cu -- exact-fp32 differential attention prefill (SIMT FFMA, accurate expf).
//
// Used for fp32 inputs (the tensor cores have no fp32-exact MMA). One warp owns one query
// row of one differential unit (V1 head or V2 pair) and walks the visible keys 32 at a
// time with two online softmaxes (one running max / sum per branch):
//   s_b[j] = q_b . k_b[j] / sqrt(d)
//   O_b    = sum_j exp(s_b[j] - m_b) v[j],  l_b = sum_j exp(s_b[j] - m_b)
//   o      = O_1 / l_1 - lambda * O_2 / l_2
//   V1:  o <- o / sqrt(mean(o^2) + eps) * (1 - lambda_init)
// ("Differential Attention (V2)", The Concept and "V1 vs V2"; "Attention Variants",
// Build It, Steps 1 and 4.) The online form is the same sum rescaled, exact up to rounding.
#include "common.cuh"
#include "kernels.h"

namespace diffattn {

namespace {
constexpr int kWarps = 4;
constexpr int kMaxD = 128;          // branch width
constexpr int kMaxDv = 2 * kMaxD;   // value width (V1: 2d)
constexpr int kPerLane = kMaxDv / 32;
}  // namespace

__global__ void __launch_bounds__(kWarps * 32) prefill_f32_kernel(PrefillArgs a) {
  __shared__ __align__(16) float qs[kWarps][2][kMaxD];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kWarps + warp;  // query row
  const int u = blockIdx.y;                  // V1 head / V2 pair
  const int b = blockIdx.z;
  // the sequence of this row (a variable-length batch packs several into one tensor)
  const SeqRange sr = seq_range(a, b);
  if (!sr.ok) {
    if (i == 0 && u == 0 && threadIdx.x == 0) report_status(a.dev_status, DIFFATTN_ERR_INVALID_ARG);
    return;
  }
  if (i >= sr.nq) return;
  const int64_t qrow = (int64_t)sr.bc * a.qs[0] + (int64_t)(sr.qrow0 + i) * a.qs[1];
  const int64_t krow0 = (int64_t)sr.bc * a.ks[0] + (int64_t)sr.krow0 * a.ks[1];
  const int64_t vrow0 = (int64_t)sr.bc * a.vs[0] + (int64_t)sr.krow0 * a.vs[1];
  const int d = a.d, dv = a.dv;
  const float* q = static_cast<const float*>(a.q);
  const float* k = static_cast<const float*>(a.k);
  const float* v = static_cast<const float*>(a.v);

  const float *q1, *q2, *k1, *k2, *vb;
  if (a.variant == DIFFATTN_V1) {
    q1 = q + qrow + u * a.qs[2];
    q2 = q1 + d;
    k1 = k + krow0 + u * a.ks[2];
    k2 = k1 + d;
    vb = v + vrow0 + u * a.vs[2];
  } else {
    const int h1 = 2 * u, h2 = 2 * u + 1;
    const int g1 = h1 / a.group, g2 = h2 / a.group;
    q1 = q + qrow + h1 * a.qs[2];
    q2 = q + qrow + h2 * a.qs[2];
    k1 = k + krow0 + g1 * a.ks[2];
    k2 = k + krow0 + g2 * a.ks[2];
    vb = v + vrow0 + g1 * a.vs[2];
  }
  const bool q_ok = in_bounds(q1 - q, d, a.ext_q, a.dev_status, a.dbg_status) &&
                    in_bounds(q2 - q, d, a.ext_q, a.dev_status, a.dbg_status);
  for (int c = lane; c < d; c += 32) {
    qs[warp][0][c] = q_ok ? q1[c] : 0.f;
    qs[warp][1][c] = q_ok ? q2[c] : 0.f;
  }
  __syncwarp();

  const float scale = 1.0f / sqrtf((float)d);
  float m1 = -INFINITY, m2 = -INFINITY, l1 = 0.f, l2 = 0.f;
  float acc1[kPerLane], acc2[kPerLane];
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) acc1[t] = acc2[t] = 0.f;

  // visible keys key_lo .. n_keys - 1: query i sits at position i + nk - nq; causal stops at
  // its own position, a sliding window keeps the last `window` of those
  const int n_keys = a.causal ? i + (sr.nk - sr.nq) + 1 : sr.nk;
  const int key_lo = (a.causal && a.window > 0) ? max(0, n_keys - a.window) : 0;
  for (int j0 = key_lo; j0 < n_keys; j0 += 32) {
    const int j = j0 + lane;
    float s1 = -INFINITY, s2 = -INFINITY;
    if (j < n_keys && in_bounds(k1 + (int64_t)j * a.ks[1] - k, d, a.ext_k, a.dev_status, a.dbg_status) &&
        in_bounds(k2 + (int64_t)j * a.ks[1] - k, d, a.ext_k, a.dev_status, a.dbg_status)) {
      const float4* kr1 = reinterpret_cast<const float4*>(k1 + (int64_t)j * a.ks[1]);
      const float4* kr2 = reinterpret_cast<const float4*>(k2 + (int64_t)j * a.ks[1]);
      const float4* qa = reinterpret_cast<const float4*>(qs[warp][0]);
      const float4* qb = reinterpret_cast<const float4*>(qs[warp][1]);
      float d1 = 0.f, d2 = 0.f;
      for (int c = 0; c < d / 4; ++c) {
        float4 x = kr1[c], y = qa[c];
        d1 = fmaf(x.x, y.x, d1); d1 = fmaf(x.y, y.y, d1);
        d1 = fmaf(x.z, y.z, d1); d1 = fmaf(x.w, y.w, d1);
        float4 z = kr2[c], w = qb[c];
        d2 = fmaf(z.x, w.x, d2); d2 = fmaf(z.y, w.y, d2);
        d2 = fmaf(z.z, w.z, d2); d2 = fmaf(z.w, w.w, d2);
      }
      s1 = d1 * scale;
      s2 = d2 * scale;
    }
    const float n1 = fmaxf(m1, warp_max(s1)), n2 = fmaxf(m2, warp_max(s2));
    const float al1 = (m1 == -INFINITY) ? 0.f : expf(m1 - n1);
    const float al2 = (m2 == -INFINITY) ? 0.f : expf(m2 - n2);
    const float p1 = (j < n_keys) ? expf(s1 - n1) : 0.f;
    const float p2 = (j < n_keys) ? expf(s2 - n2) : 0.f;
    l1 = l1 * al1 + warp_sum(p1);
    l2 = l2 * al2 + warp_sum(p2);
    m1 = n1;
    m2 = n2;
#pragma unroll
    for (int t = 0; t < kPerLane; ++t) {
      acc1[t] *= al1;
      acc2[t] *= al2;
    }
    const int jn = min(32, n_keys - j0);
    for (int jj = 0; jj < jn; ++jj) {
      const float w1 = __shfl_sync(0xffffffffu, p1, jj);
      const float w2 = __shfl_sync(0xffffffffu, p2, jj);
      const float* vr = vb + (int64_t)(j0 + jj) * a.vs[1];
      const bool v_ok = in_bounds(vr - v, dv, a.ext_v, a.dev_status, a.dbg_status);
#pragma unroll
      for (int t = 0; t < kPerLane; ++t) {
        const int c = lane + 32 * t;
        if (c < dv && v_ok) {
          const float x = vr[c];
          acc1[t] = fmaf(w1, x, acc1[t]);
          acc2[t] = fmaf(w2, x, acc2[t]);
        }
      }
    }
  }

  const float lam = a.lambda[u];
  float o[kPerLane];
  float ss = 0.f;
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    o[t] = acc1[t] / l1 - lam * (acc2[t] / l2);
    if (lane + 32 * t < dv) ss = fmaf(o[t], o[t], ss);
  }
  if (a.apply_norm) {
    ss = warp_sum(ss);
    const float r = sqrtf(ss / (float)dv + a.eps);
    const float sc = 1.0f - a.lambda_init[0];
#pragma unroll
    for (int t = 0; t < kPerLane; ++t) o[t] = o[t] / r * sc;
  }
  const int64_t o_off = (int64_t)sr.bc * a.os[0] + (int64_t)(sr.qrow0 + i) * a.os[1] + u * a.os[2];
  float* ob = static_cast<float*>(a.out) + o_off;
  const bool o_ok = in_bounds(o_off, dv, a.ext_out, a.dev_status, a.dbg_status);
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    const int c = lane + 32 * t;
    if (c < dv && o_ok) ob[c] = o[t];
  }
}

cudaError_t launch_prefill_f32(const PrefillArgs& a, cudaStream_t stream) {
  dim3 grid((a.N + kWarps - 1) / kWarps, a.units, a.B);
  prefill_f32_kernel<<<grid, kWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace diffattn
