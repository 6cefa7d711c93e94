// Producer-side fusion: causal depthwise convolution + SiLU + quantizer (or
// soft-edge encoder) in one pass, binary16 in, 8-bit codes out.
//
// In the Mamba-1 block the scan input x is produced by a short causal
// depthwise convolution along time followed by SiLU.  The Quamba-SE write-up
// (section 4.1) puts the range check -- the quantizer / soft-edge encoder --
// right where that activation is produced; Quamba2 (abstract, method step 3)
// quantizes x per sorted-and-clustered channel group.  Doing both in the
// producer removes a binary16 write and read of x through HBM.
//
// The value that is quantized is a binary32 evaluation defined step by step
// (so that a code, decided in binary32 by the quantizer's rule, is the same
// on any IEEE implementation):
//   a   = bias_c; a = fma(w[c][k], x[t - (W - 1) + k], a) for k = 0 .. W-1
//         (oldest tap first; steps before 0 read the conv state x_prev)
//   e   = exp32(-a): Cody and Waite's reduction k = rne(fl32(v log2 e)),
//         r = fma(-k, LN2_LO, fma(-k, LN2_HI, v)), the Taylor polynomial of
//         degree 7 in Horner form, times 2^k; v > 88 -> inf, v < -87 -> 0
//   u   = fl32(a * fl32(1 / fl32(1 + e)))   (IEEE reciprocal)
// then the group quantizer's or the encoder's binary32 rule on u.
//
// Layout (b, d, L), channel rows contiguous in time.  A thread takes 16
// consecutive steps of one row (two 16-byte loads) plus the 3 inputs before
// them (one 8-byte load, an L1/L2 hit: they belong to the neighbouring
// thread's vector); four CTAs of eight warps per SM hide the load latency.
// The conv taps and the exponential run as packed fp32x2
// operations (each lane a correctly rounded fma / add / multiply, so the
// packing changes no bit); the IEEE reciprocal is per element.  Vectors with
// an |a| above 87 (or a NaN) take the scalar route, which handles the range
// ends of the definition.  Rows whose length is not a multiple of 16 go
// element by element.
#include "common.cuh"
#include "internal.h"
#include "quant_fast.cuh"

namespace ssmq {
namespace {

constexpr int kConvThreads = 256;
constexpr int kConvCtasPerSm = 4;

struct ConvParams {
  int64_t b, L, d;
  int W;
  const uint16_t* x;
  const float* w;
  const float* bias;
  const uint16_t* x_prev;
  int fmt;  // SSMQ_X_INT8_GROUP or SSMQ_X_SOFTEDGE
  const int32_t* x_group;
  const float* x_scale;
  int n_groups;
  SeSteps se;
  float se_lo, se_hi;
  uint8_t* codes;
  float* u;
  uint16_t* x_prev_out;
  uint32_t* status;
};

__device__ __forceinline__ float pow2f(int k) { return __int_as_float((k + 127) << 23); }

// max that returns NaN when either operand is NaN (fmaxf would drop it)
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// The definition's e^v, scalar, every range case.
__device__ __forceinline__ float exp32(float v) {
  if (v != v) return v;
  if (v > 88.0f) return __int_as_float(0x7F800000);
  if (v < -87.0f) return 0.0f;
  const float log2e = 1.44269504088896340736f;
  const float ln2_hi = 0.693145751953125f;
  const float ln2_lo = (float)(0.69314718055994530942 - 0.693145751953125);
  const float kf = rintf(__fmul_rn(v, log2e));
  float r = __fmaf_rn(-kf, ln2_hi, v);
  r = __fmaf_rn(-kf, ln2_lo, r);
  float p = (float)(1.0 / 5040.0);
  p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  return __fmul_rn(p, pow2f((int)kf));
}

__device__ __forceinline__ float silu32(float a) {
  const float e = exp32(-a);
  return __fmul_rn(a, __frcp_rn(__fadd_rn(1.0f, e)));
}

// The same steps on a pair, for |v| <= 87 (the caller has checked): the
// rounding to an integer by the 1.5 * 2^23 sum (ties to even, exact for the
// |v log2 e| < 2^22 met here), 2^k from the sum's low bits.
__device__ __forceinline__ float2 exp32x2(float2 v) {
  const float2 log2e = make_float2(1.44269504088896340736f, 1.44269504088896340736f);
  const float2 mg = make_float2(12582912.0f, 12582912.0f);
  const float hi = 0.693145751953125f;
  const float lo = (float)(0.69314718055994530942 - 0.693145751953125);
  const float2 m = fadd2(fmul2(v, log2e), mg);
  const float2 kf = fsub2(m, mg);
  const float2 nk = make_float2(-kf.x, -kf.y);
  float2 r = ffma2(nk, make_float2(hi, hi), v);
  r = ffma2(nk, make_float2(lo, lo), r);
  const float c7 = (float)(1.0 / 5040.0), c6 = (float)(1.0 / 720.0), c5 = (float)(1.0 / 120.0);
  const float c4 = (float)(1.0 / 24.0), c3 = (float)(1.0 / 6.0);
  float2 p = make_float2(c7, c7);
  p = ffma2(p, r, make_float2(c6, c6));
  p = ffma2(p, r, make_float2(c5, c5));
  p = ffma2(p, r, make_float2(c4, c4));
  p = ffma2(p, r, make_float2(c3, c3));
  p = ffma2(p, r, make_float2(0.5f, 0.5f));
  p = ffma2(p, r, make_float2(1.0f, 1.0f));
  p = ffma2(p, r, make_float2(1.0f, 1.0f));
  // k = bits(m) - bits(1.5 * 2^23); 2^k = (k + 127) << 23
  const int kx = __float_as_int(m.x) - 0x4B400000, ky = __float_as_int(m.y) - 0x4B400000;
  return fmul2(p, make_float2(pow2f(kx), pow2f(ky)));
}

// One element of the definition: conv taps from xs[0..W) (oldest first).
__device__ __forceinline__ float conv1(const float (&xs)[4], const float (&w)[4], float bias, int W) {
  float a = bias;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k < W) a = __fmaf_rn(w[k], xs[k], a);
  return a;
}

// The code(s) of 16 values u of channel c (one group), fast route first.
__device__ __forceinline__ uint4 encode16(const ConvParams& p, const float (&u)[kQVec], float s,
                                          float rs, bool okg, uint32_t& flags) {
  uint4 o;
  if (p.fmt == SSMQ_X_INT8_GROUP) {
    if (okg && rs != 0.0f && quant16_fast(u, make_float2(s, rs), make_float2(s, rs), o)) return o;
    int r[kQVec];
#pragma unroll
    for (int i = 0; i < kQVec; ++i) r[i] = quant_elem(u[i], s, rs, okg, flags);
    o.x = pack4(r[0], r[1], r[2], r[3]);
    o.y = pack4(r[4], r[5], r[6], r[7]);
    o.z = pack4(r[8], r[9], r[10], r[11]);
    o.w = pack4(r[12], r[13], r[14], r[15]);
    return o;
  }
  const bool fast_ok = p.se.rs[0] != 0.0f && p.se.rs[1] != 0.0f && p.se.rs[2] != 0.0f;
  if (fast_ok && se16_fast(u, p.se_lo, p.se_hi, p.se, o)) return o;
  uint32_t wd[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    wd[k] = se_encode1(u[4 * k], p.se_lo, p.se_hi, p.se, flags) |
            (se_encode1(u[4 * k + 1], p.se_lo, p.se_hi, p.se, flags) << 8) |
            (se_encode1(u[4 * k + 2], p.se_lo, p.se_hi, p.se, flags) << 16) |
            (se_encode1(u[4 * k + 3], p.se_lo, p.se_hi, p.se, flags) << 24);
  return make_uint4(wd[0], wd[1], wd[2], wd[3]);
}

// Group scale of channel c and its reciprocal for the fast route (0: exact
// division only); okg false for an out-of-range id.
__device__ __forceinline__ void group_scale(const ConvParams& p, int64_t c, float& s, float& rs,
                                            bool& okg) {
  s = 0.0f;
  rs = 0.0f;
  okg = true;
  if (p.fmt != SSMQ_X_INT8_GROUP) return;
  const int g = __ldg(p.x_group + c);
  okg = (unsigned)g < (unsigned)p.n_groups;
  if (!okg) return;
  s = __ldg(p.x_scale + g);
  const float r = __frcp_rn(s);
  rs = usable_recip(s, r) ? r : 0.0f;
}

struct Raw16 {
  uint4 a, b;  // 16 binary16 steps
  uint2 h;     // the 4 steps before them (the first is unused)
};

// Vector path: rows of L % 16 == 0 steps; vector v covers steps 16 (v % (L /
// 16)) .. + 15 of row v / (L / 16).
__global__ void __launch_bounds__(kConvThreads, kConvCtasPerSm) conv_vec_kernel(const ConvParams p) {
  const int64_t vpr = p.L / 16;  // vectors per row
  const int64_t nvec = p.b * p.d * vpr;
  const int64_t stride = (int64_t)gridDim.x * kConvThreads;
  uint32_t flags = 0;
  const int S = p.W - 1;

  auto load = [&](int64_t v, Raw16& r) {
    const int64_t row = v / vpr, t0 = (v % vpr) * 16;
    const uint16_t* xr = p.x + row * p.L;
    const uint4* q = reinterpret_cast<const uint4*>(xr + t0);
    r.a = __ldg(q);
    r.b = __ldg(q + 1);
    if (t0 >= 4) {
      r.h = __ldg(reinterpret_cast<const uint2*>(xr + t0 - 4));
    } else {
      // first vector of the row: the state (times -S .. -1) or zeros
      uint16_t hv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)  // slot i holds step i - 4: state slot i - (4 - S)
        hv[i] = (p.x_prev && i >= 4 - S) ? p.x_prev[row * S + i - (4 - S)] : (uint16_t)0;
      r.h = make_uint2((uint32_t)hv[0] | ((uint32_t)hv[1] << 16),
                       (uint32_t)hv[2] | ((uint32_t)hv[3] << 16));
    }
  };

  for (int64_t v = (int64_t)blockIdx.x * kConvThreads + threadIdx.x; v < nvec; v += stride) {
    Raw16 cur;
    load(v, cur);
    const int64_t row = v / vpr, t0 = (v % vpr) * 16;
    const int64_t c = row % p.d;
    // xs[0..19]: steps t0 - 4 .. t0 + 15 (wd: the same as binary16 pairs)
    const uint32_t wd[10] = {cur.h.x, cur.h.y, cur.a.x, cur.a.y, cur.a.z, cur.a.w,
                             cur.b.x, cur.b.y, cur.b.z, cur.b.w};
    float xs[20];
#pragma unroll
    for (int i = 0; i < 10; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wd[i]));
      xs[2 * i] = f.x;
      xs[2 * i + 1] = f.y;
    }
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = k < p.W ? __ldg(p.w + c * p.W + k) : 0.0f;
    const float bias = p.bias ? __ldg(p.bias + c) : 0.0f;
    // a[i] = bias + sum_k w[k] xs[4 + i - S + k]: the taps aligned so that the
    // last one (k = W - 1) meets step t0 + i
    float a[16];
    {
      float2 acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = make_float2(bias, bias);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k < p.W) {
          const int off = 4 - S + k;  // 1..4
          const float2 wk = make_float2(w[k], w[k]);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // off is warp-uniform; select the pair without dynamic indexing
            float2 xv;
            switch (off) {
              case 1: xv = make_float2(xs[2 * j + 1], xs[2 * j + 2]); break;
              case 2: xv = make_float2(xs[2 * j + 2], xs[2 * j + 3]); break;
              case 3: xv = make_float2(xs[2 * j + 3], xs[2 * j + 4]); break;
              default: xv = make_float2(xs[2 * j + 4], xs[2 * j + 5]); break;
            }
            acc[j] = ffma2(wk, xv, acc[j]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        a[2 * j] = acc[j].x;
        a[2 * j + 1] = acc[j].y;
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmax_nan(amax, fabsf(a[i]));
    float u[16];
    if (amax <= 87.0f) {  // false for a NaN too
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 e = exp32x2(make_float2(-a[2 * j], -a[2 * j + 1]));
        const float2 den = fadd2(make_float2(1.0f, 1.0f), e);
        u[2 * j] = __fmul_rn(a[2 * j], __frcp_rn(den.x));
        u[2 * j + 1] = __fmul_rn(a[2 * j + 1], __frcp_rn(den.y));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) u[i] = silu32(a[i]);
    }
    float s, rs;
    bool okg;
    group_scale(p, c, s, rs, okg);
    const uint4 code = encode16(p, u, s, rs, okg, flags);
    const int64_t e0 = row * p.L + t0;
    *reinterpret_cast<uint4*>(p.codes + e0) = code;
    if (p.u) {
      float4* uo = reinterpret_cast<float4*>(p.u + e0);
#pragma unroll
      for (int q = 0; q < 4; ++q) uo[q] = make_float4(u[4 * q], u[4 * q + 1], u[4 * q + 2], u[4 * q + 3]);
    }
    if (p.x_prev_out && t0 + 16 == p.L) {
      // the row's last S inputs (steps L - S .. L - 1 = xs[20 - S ..])
#pragma unroll
      for (int i = 17; i < 20; ++i)  // slot j = i - (20 - S) for i >= 20 - S
        if (i >= 20 - S) p.x_prev_out[row * S + i - (20 - S)] = (uint16_t)(wd[i / 2] >> (16 * (i & 1)));
    }
  }
  flag_status(p.status, flags);
}

// Any shape: one element per thread (and the conv state of each row).
__global__ void __launch_bounds__(kConvThreads) conv_elem_kernel(const ConvParams p) {
  const int64_t n = p.b * p.d * p.L;
  const int S = p.W - 1;
  uint32_t flags = 0;
  for (int64_t e = (int64_t)blockIdx.x * kConvThreads + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * kConvThreads) {
    const int64_t row = e / p.L, t = e % p.L, c = row % p.d;
    float xs[4] = {0.0f, 0.0f, 0.0f, 0.0f}, w[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= p.W) continue;
      const int64_t sidx = t - S + k;
      if (sidx >= 0)
        xs[k] = h2f(p.x[row * p.L + sidx]);
      else if (p.x_prev)
        xs[k] = h2f(p.x_prev[row * S + S + sidx]);
      w[k] = __ldg(p.w + c * p.W + k);
    }
    const float u = silu32(conv1(xs, w, p.bias ? __ldg(p.bias + c) : 0.0f, p.W));
    float s, rs;
    bool okg;
    group_scale(p, c, s, rs, okg);
    uint32_t code;
    if (p.fmt == SSMQ_X_INT8_GROUP)
      code = (uint32_t)quant_elem(u, s, rs, okg, flags) & 0xFFu;
    else
      code = se_encode1(u, p.se_lo, p.se_hi, p.se, flags);
    p.codes[e] = (uint8_t)code;
    if (p.u) p.u[e] = u;
  }
  flag_status(p.status, flags);
}

// The conv state of every row (the path above leaves it to this kernel when
// the rows are not vectorised): slot j holds step L - S + j, or the old
// state's when L < S.
__global__ void conv_state_kernel(const ConvParams p) {
  const int S = p.W - 1;
  const int64_t n = p.b * p.d * S;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / S, j = i % S, s = p.L - S + j;
    uint16_t h = 0;
    if (s >= 0)
      h = p.x[row * p.L + s];
    else if (p.x_prev)
      h = p.x_prev[row * S + S + s];
    p.x_prev_out[i] = h;
  }
}

}  // namespace

cudaError_t launch_conv_silu_quantize(const ssmq_conv_args& a, cudaStream_t st) {
  ConvParams p{};
  p.b = a.batch;
  p.L = a.seqlen;
  p.d = a.dim;
  p.W = a.width;
  p.x = a.x;
  p.w = a.weight;
  p.bias = a.bias;
  p.x_prev = a.x_prev;
  p.fmt = a.out_format;
  p.x_group = a.x_group;
  p.x_scale = a.x_scale;
  p.n_groups = a.n_x_groups;
  p.se = se_steps(a.se_scale, a.se_log2_ratio);
  p.se_lo = a.se_lo;
  p.se_hi = a.se_hi;
  p.codes = static_cast<uint8_t*>(a.codes);
  p.u = a.u;
  p.x_prev_out = a.x_prev_out;
  p.status = a.status;
  const int sms = sm_count();
  const int64_t n = p.b * p.d * p.L;
  const bool vec = p.L > 0 && p.L % 16 == 0;
  if (n > 0) {
    if (vec) {
      const int64_t nvec = n / 16;
      int64_t grid = (nvec + kConvThreads - 1) / kConvThreads;
      grid = grid < (int64_t)sms * kConvCtasPerSm ? grid : (int64_t)sms * kConvCtasPerSm;
      conv_vec_kernel<<<(unsigned)grid, kConvThreads, 0, st>>>(p);
    } else {
      int64_t grid = (n + kConvThreads - 1) / kConvThreads;
      grid = grid < (int64_t)sms * 8 ? grid : (int64_t)sms * 8;
      conv_elem_kernel<<<(unsigned)grid, kConvThreads, 0, st>>>(p);
    }
  }
  if (p.x_prev_out && p.W > 1 && !vec) {
    const int64_t ns = p.b * p.d * (p.W - 1);
    if (ns > 0) {
      int64_t grid = (ns + 255) / 256;
      grid = grid < (int64_t)sms * 8 ? grid : (int64_t)sms * 8;
      conv_state_kernel<<<(unsigned)grid, 256, 0, st>>>(p);
    }
  }
  return cudaGetLastError();
}

}  // namespace ssmq
