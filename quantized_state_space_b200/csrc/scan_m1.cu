// Mamba-1 diagonal selective scan on W8A8 operands (sm_100a).
//
// Quamba2 (shd-paper.top card), abstract: W8A8 for the Mamba1 backbone -- the
// inputs of the linear recurrence are 8-bit: x per sorted-and-clustered
// channel group, B and C per state group, each with an fp32 scale.  The
// recurrence per (batch b, channel c, state n):
//     h_t = exp(delta_t A_cn) h_{t-1} + delta_t B_tn x_t
//     y_t = sum_n C_tn h_tn + D_c x_t,   y_t *= silu(z_t) when gated
// Quamba-SE write-up 2.2: x may instead arrive as soft-edge byte codes, which
// are decoded in registers here (the scan reads one byte per element either
// way).
//
// Work decomposition.  Every (b, c, n) recurrence is owned by one thread from
// t = 0 to L - 1, so each decay exp(delta A) is evaluated exactly once and no
// carry pass is needed.  A CTA owns kCH channels of one batch row and one B/C
// group and walks L in chunks of kT = 64 steps:
//   phase A  all threads stage the chunk: 16-byte loads of x codes and of
//            binary16 dt / z, dequantisation, softplus, silu, D x; B and C
//            rows are loaded as int8, dequantised once per (t, n) and
//            transposed into shared memory as [t][n] fp32 (shared by all
//            channels of the CTA);
//   phase B  thread (c, j) advances states 4j..4j+3 of channel c through the
//            chunk: one MUFU.EX2 per state update, the rest FMA; the
//            per-thread partial sums of C . h are combined across the
//            N / 4 threads of a channel by a shuffle reduce-scatter, so each
//            thread ends up owning the full y of one time step;
//   phase C  all threads apply (y + D x) * silu(z) and store binary16 y with
//            16-byte stores.
// The state stays in registers across chunks; the final state is written once.
#include "common.cuh"
#include "internal.h"

namespace ssmq {
namespace {

constexpr int kT = 64;    // time steps per chunk
constexpr int kSeg = 16;  // time steps per staging work item
constexpr int kSPL = 4;   // states per thread

struct M1Params {
  int64_t b, L, d, G;
  int gs;
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
  const float* h0;
  uint16_t* y;
  float* h_final;
  uint32_t* status;
  int n_ctile;
  int vec_ok;
};

__device__ __forceinline__ void load_u8x16(const uint8_t* p, int cnt, bool vec, uint8_t (&o)[16]) {
  if (vec && cnt == 16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = (uint8_t)(w[i >> 2] >> (8 * (i & 3)));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = i < cnt ? p[i] : (uint8_t)0;
  }
}

__device__ __forceinline__ void load_h16(const uint16_t* p, int cnt, bool vec, uint16_t (&o)[16]) {
  if (vec && cnt == 16) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = (uint16_t)(w[i >> 1] >> (16 * (i & 1)));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = i < cnt ? p[i] : (uint16_t)0;
  }
}

// Reduce-scatter over the LPC consecutive lanes of a channel: on entry each
// lane holds LPC partial sums (one per time step of the group); on exit lane
// j returns the sum over the LPC lanes of entry j.
template <int LPC>
__device__ __forceinline__ float reduce_scatter(float (&p)[LPC], int j) {
#pragma unroll
  for (int w = LPC / 2; w >= 1; w /= 2) {
    const bool upper = (j & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float keep = upper ? p[i + w] : p[i];
      const float send = upper ? p[i] : p[i + w];
      p[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return p[0];
}

template <int kN, int kCH, int kXFmt>
__global__ void __launch_bounds__(kCH * (kN / kSPL))
    m1_scan_kernel(const M1Params p) {
  constexpr int LPC = kN / kSPL;
  constexpr int NT = kCH * LPC;
  constexpr int RW = kT + 1;   // float2 row: conflict-free column reads in phase B
  constexpr int RY = kT + 4;   // float row of the reduced sums
  constexpr int SEGS = kT / kSeg;
  __shared__ float2 sDD[kCH][RW];  // (delta, delta * x)
  __shared__ float2 sEP[kCH][RW];  // (D * x, silu(z) or 1)
  __shared__ __align__(16) float sB[kT][kN];
  __shared__ __align__(16) float sC[kT][kN];
  __shared__ float sY[kCH][RY];

  const int tid = threadIdx.x;
  const int64_t bb = blockIdx.y;
  const int64_t d = p.d, L = p.L;
  const int dg = (int)(d / p.G);
  const int g = blockIdx.x / p.n_ctile;
  const int c0 = g * dg + (blockIdx.x % p.n_ctile) * kCH;
  const int nc = min(kCH, g * dg + dg - c0);
  const int spg = kN / p.gs;
  const bool vec = p.vec_ok != 0;
  uint32_t flags = 0;

  // scan role
  const int lc = tid / LPC, lj = tid % LPC;
  const bool lvalid = lc < nc;
  const int64_t lch = c0 + lc;
  float h[kSPL], a2[kSPL];
#pragma unroll
  for (int s = 0; s < kSPL; ++s) {
    const int n = lj * kSPL + s;
    a2[s] = lvalid ? __ldg(p.A + lch * kN + n) * kLog2e : 0.0f;
    h[s] = (lvalid && p.h0) ? __ldg(p.h0 + (bb * d + lch) * kN + n) : 0.0f;
  }

  for (int64_t t0 = 0; t0 < L; t0 += kT) {
    const int tl = (int)min((int64_t)kT, L - t0);

    // ---- phase A: x, dt, z -> (delta, delta x) and (D x, gate)
    for (int w = tid; w < kCH * SEGS; w += NT) {
      const int c = w / SEGS, tb = (w % SEGS) * kSeg;
      float2 dd[kSeg], ep[kSeg];
      if (c < nc && tb < tl) {
        const int64_t ch = c0 + c;
        const int64_t row = (bb * d + ch) * L + t0 + tb;
        const int cnt = min(kSeg, tl - tb);
        uint8_t xq[kSeg];
        uint16_t dtb[kSeg], zb[kSeg];
        load_u8x16(static_cast<const uint8_t*>(p.x) + row, cnt, vec, xq);
        load_h16(p.dt + row, cnt, vec, dtb);
        if (p.z) load_h16(p.z + row, cnt, vec, zb);
        float xs = 1.0f;
        if (kXFmt == SSMQ_X_INT8_GROUP) {
          const int xg = __ldg(p.x_group + ch);
          if ((unsigned)xg < (unsigned)p.n_x_groups) {
            xs = __ldg(p.x_scale + xg);
          } else {
            xs = 0.0f;
            flags |= SSMQ_DEV_BAD_GROUP;
          }
        }
        const float bias = p.dt_bias ? __ldg(p.dt_bias + ch) : 0.0f;
        const float Dc = p.D ? __ldg(p.D + ch) : 0.0f;
#pragma unroll
        for (int i = 0; i < kSeg; ++i) {
          float xv;
          if (kXFmt == SSMQ_X_INT8_GROUP)
            xv = (float)(int8_t)xq[i] * xs;
          else
            xv = se_decode(xq[i], p.se);
          const float dv = h2f(dtb[i]) + bias;
          float delta = p.softplus ? softplus_f(dv) : dv;
          if (i >= cnt) delta = 0.0f;
          dd[i] = make_float2(delta, delta * xv);
          ep[i] = make_float2(Dc * xv, p.z ? silu_f(h2f(zb[i])) : 1.0f);
        }
      } else {
#pragma unroll
        for (int i = 0; i < kSeg; ++i) {
          dd[i] = make_float2(0.0f, 0.0f);
          ep[i] = make_float2(0.0f, 0.0f);
        }
      }
#pragma unroll
      for (int i = 0; i < kSeg; ++i) {
        sDD[c][tb + i] = dd[i];
        sEP[c][tb + i] = ep[i];
      }
    }
    // ---- phase A: B and C rows of group g -> [t][n] fp32
    for (int w = tid; w < 2 * kN * SEGS; w += NT) {
      const int which = w / (kN * SEGS);
      const int rem = w % (kN * SEGS);
      const int n = rem / SEGS, tb = (rem % SEGS) * kSeg;
      const int cnt = max(0, min(kSeg, tl - tb));
      const int8_t* base = which ? p.C : p.B;
      const float sc = __ldg((which ? p.C_scale : p.B_scale) + g * spg + n / p.gs);
      uint8_t q[kSeg];
      if (cnt > 0)
        load_u8x16(reinterpret_cast<const uint8_t*>(base) + ((bb * p.G + g) * kN + n) * L + t0 + tb,
                   cnt, vec, q);
      else
#pragma unroll
        for (int i = 0; i < kSeg; ++i) q[i] = 0;
      float* dst = which ? &sC[0][0] : &sB[0][0];
#pragma unroll
      for (int i = 0; i < kSeg; ++i) dst[(tb + i) * kN + n] = (float)(int8_t)q[i] * sc;
    }
    __syncthreads();

    // ---- phase B: the recurrence, one thread per 4 states of a channel
#pragma unroll 1
    for (int tg = 0; tg < kT / LPC; ++tg) {
      float part[LPC];
#pragma unroll
      for (int k = 0; k < LPC; ++k) {
        const int t = tg * LPC + k;
        const float2 dd = sDD[lc][t];
        const float4 b4 = *reinterpret_cast<const float4*>(&sB[t][lj * kSPL]);
        const float4 c4 = *reinterpret_cast<const float4*>(&sC[t][lj * kSPL]);
        const float e0 = ex2_sfu(dd.x * a2[0]);
        const float e1 = ex2_sfu(dd.x * a2[1]);
        const float e2 = ex2_sfu(dd.x * a2[2]);
        const float e3 = ex2_sfu(dd.x * a2[3]);
        h[0] = fmaf(e0, h[0], dd.y * b4.x);
        h[1] = fmaf(e1, h[1], dd.y * b4.y);
        h[2] = fmaf(e2, h[2], dd.y * b4.z);
        h[3] = fmaf(e3, h[3], dd.y * b4.w);
        part[k] = fmaf(c4.x, h[0], fmaf(c4.y, h[1], fmaf(c4.z, h[2], c4.w * h[3])));
      }
      sY[lc][tg * LPC + lj] = reduce_scatter<LPC>(part, lj);
    }
    __syncthreads();

    // ---- phase C: epilogue and binary16 stores
    for (int w = tid; w < kCH * SEGS; w += NT) {
      const int c = w / SEGS, tb = (w % SEGS) * kSeg;
      if (c < nc && tb < tl) {
        const int cnt = min(kSeg, tl - tb);
        uint16_t* dst = p.y + (bb * d + c0 + c) * L + t0 + tb;
        uint32_t wv[kSeg / 2];
#pragma unroll
        for (int i = 0; i < kSeg; i += 2) {
          const float2 e0 = sEP[c][tb + i], e1 = sEP[c][tb + i + 1];
          const float y0 = (sY[c][tb + i] + e0.x) * e0.y;
          const float y1 = (sY[c][tb + i + 1] + e1.x) * e1.y;
          wv[i / 2] = (uint32_t)f2h(y0) | ((uint32_t)f2h(y1) << 16);
        }
        if (vec && cnt == kSeg) {
          uint4* o = reinterpret_cast<uint4*>(dst);
          o[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          o[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
        } else {
          for (int i = 0; i < cnt; ++i) dst[i] = (uint16_t)(wv[i / 2] >> (16 * (i & 1)));
        }
      }
    }
    __syncthreads();
  }

  if (lvalid && p.h_final)
    *reinterpret_cast<float4*>(p.h_final + (bb * d + lch) * kN + lj * kSPL) =
        make_float4(h[0], h[1], h[2], h[3]);
  flag_status(p.status, flags);
}

template <int kN, int kCH>
cudaError_t launch_m1(const M1Params& prm, int xfmt, int64_t batch, cudaStream_t st) {
  M1Params p = prm;
  const int dg = (int)(p.d / p.G);
  p.n_ctile = (dg + kCH - 1) / kCH;
  const dim3 grid((unsigned)(p.n_ctile * p.G), (unsigned)batch);
  const dim3 block(kCH * (kN / kSPL));
  if (xfmt == SSMQ_X_SOFTEDGE)
    m1_scan_kernel<kN, kCH, SSMQ_X_SOFTEDGE><<<grid, block, 0, st>>>(p);
  else
    m1_scan_kernel<kN, kCH, SSMQ_X_INT8_GROUP><<<grid, block, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_selective_scan(const ssmq_scan_args& a, cudaStream_t st) {
  if (a.batch == 0 || a.dim == 0) return cudaSuccess;
  M1Params p{};
  p.b = a.batch;
  p.L = a.seqlen;
  p.d = a.dim;
  p.G = a.ngroups;
  p.gs = a.state_group_size;
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
  p.h0 = a.h0;
  p.y = a.y;
  p.h_final = a.h_final;
  p.status = a.status;
  p.vec_ok = (a.seqlen % 16 == 0) ? 1 : 0;
  if (a.seqlen == 0) {
    // nothing to scan: the final state is the initial state
    if (a.h_final) {
      const size_t bytes = sizeof(float) * (size_t)(a.batch * a.dim * a.dstate);
      return a.h0 ? cudaMemcpyAsync(a.h_final, a.h0, bytes, cudaMemcpyDeviceToDevice, st)
                  : cudaMemsetAsync(a.h_final, 0, bytes, st);
    }
    return cudaSuccess;
  }
  switch (a.dstate) {
    case 4: return launch_m1<4, 32>(p, a.x_format, a.batch, st);
    case 8: return launch_m1<8, 32>(p, a.x_format, a.batch, st);
    case 16: return launch_m1<16, 16>(p, a.x_format, a.batch, st);
    case 32: return launch_m1<32, 16>(p, a.x_format, a.batch, st);
    case 64: return launch_m1<64, 8>(p, a.x_format, a.batch, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ssmq
