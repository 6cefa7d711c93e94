// Single-token decode state update, Mamba-2 form (sm_100a).
//
// Quamba2 (shd-paper.top card), abstract: the generation stage of W8A8 Mamba2
// models.  One step of the recurrence on the persistent fp32 state, per
// (batch b, head h): delta = softplus(dt + bias), dA = exp(delta A_h), and for
// every (p, n):  h_pn <- dA h_pn + delta x_p B_n,  y_p = sum_n C_n h_pn + D x_p
// (times silu(z_p) when gated).
//
// The state (b, H, P, N) fp32 is read once and written once in place, so the
// kernel is HBM-bound: one CTA per (b, h) streams its P x N tile with 16-byte
// loads and stores, N / 4 lanes per row, several rows in flight per thread;
// C . h is reduced across the row's lanes with shuffles.
#include "common.cuh"
#include "internal.h"

namespace ssmq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct DecParams {
  int64_t H, P, G;
  int gs;
  int xfmt;
  const void* x;
  const int32_t* x_group;
  const float* x_scale;
  int n_x_groups;
  SeSteps se;
  const uint16_t* dt;
  const float* dt_bias;
  int softplus;
  const float* A;
  const float* D;
  const uint16_t* z;
  const int8_t* B;
  const int8_t* C;
  const float* B_scale;
  const float* C_scale;
  float* state;
  uint16_t* y;
  uint32_t* status;
};

template <int kN>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecParams p) {
  constexpr int LPR = kN / 4;            // lanes per state row
  constexpr int RPP = kThreads / LPR;    // rows per pass
  const int64_t u = blockIdx.x;          // b * H + h
  const int64_t H = p.H, P = p.P;
  const int64_t bb = u / H, hd = u % H;
  const int64_t g = hd * p.G / H;
  const int tid = threadIdx.x, r = tid / LPR, j = tid % LPR;
  const int spg = kN / p.gs;
  uint32_t flags = 0;

  const float dv = h2f(p.dt[u]) + (p.dt_bias ? __ldg(p.dt_bias + hd) : 0.0f);
  const float delta = p.softplus ? softplus_f(dv) : dv;
  const float dA = ex2_sfu(delta * __ldg(p.A + hd) * kLog2e);
  const float Dh = p.D ? __ldg(p.D + hd) : 0.0f;

  float bv[4], cv[4];
  {
    const int64_t bo = (bb * p.G + g) * kN + j * 4;
    const char4 bq = *reinterpret_cast<const char4*>(p.B + bo);
    const char4 cq = *reinterpret_cast<const char4*>(p.C + bo);
    const int8_t bqa[4] = {bq.x, bq.y, bq.z, bq.w};
    const int8_t cqa[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int si = (int)g * spg + (j * 4 + s) / p.gs;
      bv[s] = (float)bqa[s] * __ldg(p.B_scale + si);
      cv[s] = (float)cqa[s] * __ldg(p.C_scale + si);
    }
  }

  float* st = p.state + u * P * kN;
  for (int64_t p0 = 0; p0 < P; p0 += (int64_t)RPP * kUnroll) {
    float4 hv[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t row = p0 + k * RPP + r;
      hv[k] = row < P ? *reinterpret_cast<const float4*>(st + row * kN + j * 4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t row = p0 + k * RPP + r;
      const bool ok = row < P;
      float xv = 0.0f;
      if (ok) {
        const int64_t xi = u * P + row;
        if (p.xfmt == SSMQ_X_SOFTEDGE) {
          xv = se_decode(static_cast<const uint8_t*>(p.x)[xi], p.se);
        } else {
          const int xg = __ldg(p.x_group + hd * P + row);
          if ((unsigned)xg < (unsigned)p.n_x_groups) {
            xv = (float)static_cast<const int8_t*>(p.x)[xi] * __ldg(p.x_scale + xg);
          } else {
            flags |= SSMQ_DEV_BAD_GROUP;
          }
        }
      }
      const float dx = delta * xv;
      float4 h = hv[k];
      h.x = fmaf(dA, h.x, dx * bv[0]);
      h.y = fmaf(dA, h.y, dx * bv[1]);
      h.z = fmaf(dA, h.z, dx * bv[2]);
      h.w = fmaf(dA, h.w, dx * bv[3]);
      float part = fmaf(cv[0], h.x, fmaf(cv[1], h.y, fmaf(cv[2], h.z, cv[3] * h.w)));
#pragma unroll
      for (int off = LPR / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (ok) {
        *reinterpret_cast<float4*>(st + row * kN + j * 4) = h;
        if (j == 0) {
          float yv = part + Dh * xv;
          if (p.z) yv *= silu_f(h2f(p.z[u * P + row]));
          p.y[u * P + row] = f2h(yv);
        }
      }
    }
  }
  flag_status(p.status, flags);
}

}  // namespace

cudaError_t launch_state_update(const ssmq_decode_args& a, cudaStream_t st) {
  const int64_t units = a.batch * a.nheads;
  if (units == 0 || a.headdim == 0) return cudaSuccess;
  DecParams p{};
  p.H = a.nheads;
  p.P = a.headdim;
  p.G = a.ngroups;
  p.gs = a.state_group_size;
  p.xfmt = a.x_format;
  p.x = a.x;
  p.x_group = a.x_group;
  p.x_scale = a.x_scale;
  p.n_x_groups = a.n_x_groups;
  p.se = se_steps(a.se_scale, a.se_log2_ratio);
  p.dt = a.dt;
  p.dt_bias = a.dt_bias;
  p.softplus = a.dt_softplus;
  p.A = a.A;
  p.D = a.D;
  p.z = a.z;
  p.B = a.B;
  p.C = a.C;
  p.B_scale = a.B_scale;
  p.C_scale = a.C_scale;
  p.state = a.state;
  p.y = a.y;
  p.status = a.status;
  const unsigned grid = (unsigned)units;
  switch (a.dstate) {
    case 16: decode_kernel<16><<<grid, kThreads, 0, st>>>(p); break;
    case 32: decode_kernel<32><<<grid, kThreads, 0, st>>>(p); break;
    case 64: decode_kernel<64><<<grid, kThreads, 0, st>>>(p); break;
    case 128: decode_kernel<128><<<grid, kThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ssmq

// ---------------------------------------------------------------------------
// Mamba-1 form: A per (channel, state).  One thread per 4 states of a
// (batch, channel); the N / 4 threads of a channel reduce C . h with
// shuffles.  The state (b, d, N) is read and written once with 16-byte
// accesses.
namespace ssmq {
namespace {

struct M1DecParams {
  int64_t units;  // b * d
  int64_t d, G;
  int gs;
  int xfmt;
  const void* x;
  const int32_t* x_group;
  const float* x_scale;
  int n_x_groups;
  SeSteps se;
  const uint16_t* dt;
  const float* dt_bias;
  int softplus;
  const float* A;
  const float* D;
  const uint16_t* z;
  const int8_t* B;
  const int8_t* C;
  const float* B_scale;
  const float* C_scale;
  float* state;
  uint16_t* y;
  uint32_t* status;
};

template <int kN>
__global__ void __launch_bounds__(256) m1_decode_kernel(const M1DecParams p) {
  constexpr int LPC = kN / 4;
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t u = gt / LPC;  // b * d + c
  const int j = (int)(gt % LPC);
  const bool ok = u < p.units;
  uint32_t flags = 0;
  float part = 0.0f, xv = 0.0f;
  int64_t c = 0;
  if (ok) {
    const int64_t bb = u / p.d;
    c = u % p.d;
    const int64_t g = c * p.G / p.d;
    const int spg = kN / p.gs;
    if (p.xfmt == SSMQ_X_SOFTEDGE) {
      xv = se_decode(static_cast<const uint8_t*>(p.x)[u], p.se);
    } else {
      const int xg = __ldg(p.x_group + c);
      if ((unsigned)xg < (unsigned)p.n_x_groups)
        xv = (float)static_cast<const int8_t*>(p.x)[u] * __ldg(p.x_scale + xg);
      else
        flags |= SSMQ_DEV_BAD_GROUP;
    }
    const float dv = h2f(p.dt[u]) + (p.dt_bias ? __ldg(p.dt_bias + c) : 0.0f);
    const float delta = p.softplus ? softplus_f(dv) : dv;
    const float dx = delta * xv;
    const float4 a = __ldg(reinterpret_cast<const float4*>(p.A + c * kN) + j);
    float4 h = *(reinterpret_cast<const float4*>(p.state + u * kN) + j);
    const int64_t bo = (bb * p.G + g) * kN + 4 * j;
    const char4 bq = *reinterpret_cast<const char4*>(p.B + bo);
    const char4 cq = *reinterpret_cast<const char4*>(p.C + bo);
    const float av[4] = {a.x, a.y, a.z, a.w};
    const int8_t bqa[4] = {bq.x, bq.y, bq.z, bq.w};
    const int8_t cqa[4] = {cq.x, cq.y, cq.z, cq.w};
    float hv[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int si = (int)g * spg + (4 * j + s) / p.gs;
      const float bvv = (float)bqa[s] * __ldg(p.B_scale + si);
      const float cvv = (float)cqa[s] * __ldg(p.C_scale + si);
      hv[s] = fmaf(ex2_sfu(delta * av[s] * kLog2e), hv[s], dx * bvv);
      part = fmaf(cvv, hv[s], part);
    }
    *(reinterpret_cast<float4*>(p.state + u * kN) + j) = make_float4(hv[0], hv[1], hv[2], hv[3]);
  }
#pragma unroll
  for (int off = LPC / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if (ok && j == 0) {
    float yv = part + (p.D ? __ldg(p.D + c) : 0.0f) * xv;
    if (p.z) yv *= silu_f(h2f(p.z[u]));
    p.y[u] = f2h(yv);
  }
  flag_status(p.status, flags);
}

}  // namespace

cudaError_t launch_m1_state_update(const ssmq_m1_decode_args& a, cudaStream_t st) {
  const int64_t units = a.batch * a.dim;
  if (units == 0) return cudaSuccess;
  M1DecParams p{};
  p.units = units;
  p.d = a.dim;
  p.G = a.ngroups;
  p.gs = a.state_group_size;
  p.xfmt = a.x_format;
  p.x = a.x;
  p.x_group = a.x_group;
  p.x_scale = a.x_scale;
  p.n_x_groups = a.n_x_groups;
  p.se = se_steps(a.se_scale, a.se_log2_ratio);
  p.dt = a.dt;
  p.dt_bias = a.dt_bias;
  p.softplus = a.dt_softplus;
  p.A = a.A;
  p.D = a.D;
  p.z = a.z;
  p.B = a.B;
  p.C = a.C;
  p.B_scale = a.B_scale;
  p.C_scale = a.C_scale;
  p.state = a.state;
  p.y = a.y;
  p.status = a.status;
  const int64_t threads = units * (a.dstate / 4);
  const unsigned grid = (unsigned)((threads + 255) / 256);
  switch (a.dstate) {
    case 4: m1_decode_kernel<4><<<grid, 256, 0, st>>>(p); break;
    case 8: m1_decode_kernel<8><<<grid, 256, 0, st>>>(p); break;
    case 16: m1_decode_kernel<16><<<grid, 256, 0, st>>>(p); break;
    case 32: m1_decode_kernel<32><<<grid, 256, 0, st>>>(p); break;
    case 64: m1_decode_kernel<64><<<grid, 256, 0, st>>>(p); break;
    case 128: m1_decode_kernel<128><<<grid, 256, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ssmq
