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
// group and walks L in chunks of kT = 64 steps.  The raw bytes of chunk k + 1
// (x codes, binary16 dt / z, int8 B / C rows) are fetched with cp.async into
// a second shared-memory buffer while chunk k is scanned, so the recurrence
// never waits on global memory.  Per chunk:
//   stage    all threads turn the raw bytes of the chunk into (delta, delta x)
//            per (c, t) and dequantised B, C rows laid out [t][n] (shared by
//            every channel of the CTA);
//   scan     thread (c, j) advances states 4j..4j+3 of channel c: one
//            MUFU.EX2 per state update and packed fp32x2 FMA for the rest;
//            the per-thread partial sums of C . h are combined across the
//            N / 4 threads of a channel by a shuffle reduce-scatter, so each
//            thread ends up owning the full y of one time step;
//   store    all threads apply (y + D x) * silu(z) from the raw bytes and
//            store binary16 y with 16-byte stores.
// The state stays in registers across chunks; the final state is written once.
#include "common.cuh"
#include "internal.h"

namespace ssmq {
namespace {

constexpr int kT = 64;    // time steps per chunk
constexpr int kSeg = 16;  // time steps per staging work item (16 bytes of codes)

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

// ---- cp.async (16-byte, L2-only) -------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

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

// Raw bytes of one chunk, as fetched from global memory.
template <int kN, int kCH>
struct Raw {
  uint8_t x[kCH][kT];
  uint16_t dt[kCH][kT];
  uint16_t z[kCH][kT];
  int8_t B[kN][kT];
  int8_t C[kN][kT];
};

template <int kN, int kCH>
struct M1Smem {
  Raw<kN, kCH> raw[2];                  // double-buffered raw bytes
  __align__(16) float2 dd[kCH][kT + 2]; // (delta, delta x); 16-byte rows
  __align__(16) float b[kT][kN];        // dequantised B, [t][n]
  __align__(16) float c[kT][kN];        // dequantised C, [t][n]
  float y[kCH][kT + 4];                 // C . h per (c, t)
};

template <int kN, int kCH>
__device__ __forceinline__ void fetch_chunk(const M1Params& p, Raw<kN, kCH>& r, int64_t bb, int g,
                                            int c0, int nc, int64_t t0, int tl, int tid, int NT) {
  constexpr int SEGS = kT / kSeg;
  const int64_t d = p.d, L = p.L;
  if (p.vec_ok) {
    // every row starts 16-byte aligned (L % 16 == 0): 16-byte cp.async pieces
    for (int w = tid; w < kCH * SEGS; w += NT) {
      const int c = w / SEGS, tb = (w % SEGS) * kSeg;
      if (c >= nc || tb >= tl) continue;
      const int64_t row = (bb * d + c0 + c) * L + t0 + tb;
      cp_async16(&r.x[c][tb], static_cast<const uint8_t*>(p.x) + row);
      cp_async16(&r.dt[c][tb], p.dt + row);
      cp_async16(&r.dt[c][tb + 8], p.dt + row + 8);
      if (p.z) {
        cp_async16(&r.z[c][tb], p.z + row);
        cp_async16(&r.z[c][tb + 8], p.z + row + 8);
      }
    }
    for (int w = tid; w < 2 * kN * SEGS; w += NT) {
      const int which = w / (kN * SEGS), rem = w % (kN * SEGS);
      const int n = rem % kN, tb = (rem / kN) * kSeg;
      if (tb >= tl) continue;
      const int64_t row = ((bb * p.G + g) * kN + n) * L + t0 + tb;
      cp_async16(which ? &r.C[n][tb] : &r.B[n][tb], (which ? p.C : p.B) + row);
    }
  } else {
    // rows not 16-byte aligned: plain element loads, bounded by the row end
    for (int w = tid; w < kCH * kT; w += NT) {
      const int c = w / kT, t = w % kT;
      if (c >= nc || t >= tl) continue;
      const int64_t row = (bb * d + c0 + c) * L + t0 + t;
      r.x[c][t] = static_cast<const uint8_t*>(p.x)[row];
      r.dt[c][t] = p.dt[row];
      if (p.z) r.z[c][t] = p.z[row];
    }
    for (int w = tid; w < 2 * kN * kT; w += NT) {
      const int which = w / (kN * kT), rem = w % (kN * kT);
      const int n = rem / kT, t = rem % kT;
      if (t >= tl) continue;
      const int64_t row = ((bb * p.G + g) * kN + n) * L + t0 + t;
      (which ? r.C : r.B)[n][t] = (which ? p.C : p.B)[row];
    }
  }
}

template <int kN, int kCH, int kSPL, int kXFmt>
__global__ void __launch_bounds__(kCH * (kN / kSPL))
    m1_scan_kernel(const M1Params p) {
  static_assert(kSPL == 2 || kSPL == 4, "2 or 4 states per thread");
  constexpr int NP = kSPL / 2;  // fp32x2 pairs per thread
  constexpr int LPC = kN / kSPL;
  constexpr int NT = kCH * LPC;
  constexpr int RW = kT + 2;   // float2 row: 16-byte aligned, conflict-free column reads
  constexpr int RY = kT + 4;   // float row of the reduced sums
  constexpr int SEGS = kT / kSeg;
  extern __shared__ __align__(16) uint8_t smem_bytes[];
  M1Smem<kN, kCH>& S = *reinterpret_cast<M1Smem<kN, kCH>*>(smem_bytes);
  Raw<kN, kCH>* raw = S.raw;
  float2 (*sDD)[RW] = S.dd;  // (delta, delta * x)
  float (*sB)[kN] = S.b;
  float (*sC)[kN] = S.c;
  float (*sY)[RY] = S.y;

  const int tid = threadIdx.x;
  const int64_t bb = blockIdx.y;
  const int64_t d = p.d, L = p.L;
  const int dg = (int)(d / p.G);
  const int g = blockIdx.x / p.n_ctile;
  const int c0 = g * dg + (blockIdx.x % p.n_ctile) * kCH;
  const int nc = min(kCH, g * dg + dg - c0);
  const int spg = kN / p.gs;
  uint32_t flags = 0;

  // scan role: channel lc, states 4 lj .. 4 lj + 3
  const int lc = tid / LPC, lj = tid % LPC;
  const bool lvalid = lc < nc;
  const int64_t lch = c0 + lc;
  float2 hp[NP], ap[NP];  // states 2i, 2i+1 of this thread's block of kSPL
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const int n = lj * kSPL + 2 * i;
    ap[i] = lvalid ? make_float2(__ldg(p.A + lch * kN + n) * kLog2e, __ldg(p.A + lch * kN + n + 1) * kLog2e)
                   : make_float2(0.0f, 0.0f);
    hp[i] = (lvalid && p.h0) ? make_float2(__ldg(p.h0 + (bb * d + lch) * kN + n),
                                           __ldg(p.h0 + (bb * d + lch) * kN + n + 1))
                             : make_float2(0.0f, 0.0f);
  }

  // per-channel constants of the staging role (item c = w / SEGS is fixed
  // across chunks when NT is a multiple of kCH * SEGS or larger)
  const int nchunks = (int)((L + kT - 1) / kT);
  fetch_chunk<kN, kCH>(p, raw[0], bb, g, c0, nc, 0, (int)min((int64_t)kT, L), tid, NT);
  cp_async_commit();

  // y = (C . h + D x) * silu(z) of chunk kk, binary16, from its raw bytes
  auto store_chunk = [&](int kk) {
    const int64_t t0 = (int64_t)kk * kT;
    const int tl = (int)min((int64_t)kT, L - t0);
    Raw<kN, kCH>& r = raw[kk & 1];
    for (int w = tid; w < kCH * SEGS; w += NT) {
      const int c = w / SEGS, tb = (w % SEGS) * kSeg;
      if (c >= nc || tb >= tl) continue;
      const int64_t ch = c0 + c;
      float xs = 1.0f;
      if (kXFmt == SSMQ_X_INT8_GROUP) {
        const int xg = __ldg(p.x_group + ch);
        xs = (unsigned)xg < (unsigned)p.n_x_groups ? __ldg(p.x_scale + xg) : 0.0f;
      }
      const float Dc = p.D ? __ldg(p.D + ch) : 0.0f;
      const int cnt = min(kSeg, tl - tb);
      const uint4 xw = *reinterpret_cast<const uint4*>(&r.x[c][tb]);
      const uint32_t xb[4] = {xw.x, xw.y, xw.z, xw.w};
      uint32_t zw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (p.z) {
        const uint4 z0 = *reinterpret_cast<const uint4*>(&r.z[c][tb]);
        const uint4 z1 = *reinterpret_cast<const uint4*>(&r.z[c][tb + 8]);
        zw[0] = z0.x; zw[1] = z0.y; zw[2] = z0.z; zw[3] = z0.w;
        zw[4] = z1.x; zw[5] = z1.y; zw[6] = z1.z; zw[7] = z1.w;
      }
      uint32_t wv[kSeg / 2];
#pragma unroll
      for (int i = 0; i < kSeg; i += 2) {
        float yv[2];
        const float2 zf = __half22float2(*reinterpret_cast<const __half2*>(&zw[i >> 1]));
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = i + e;
          const uint32_t code = (xb[t >> 2] >> (8 * (t & 3))) & 0xFFu;
          const float xv = kXFmt == SSMQ_X_INT8_GROUP ? s8_to_f32(xb[t >> 2] ^ 0x80808080u, t & 3) * xs
                                                      : se_decode(code, p.se);
          float v = fmaf(Dc, xv, sY[c][tb + t]);
          if (p.z) v *= silu_f(e ? zf.y : zf.x);
          yv[e] = v;
        }
        wv[i / 2] = pack_half2(yv[0], yv[1]);
      }
      uint16_t* dst = p.y + (bb * d + ch) * L + t0 + tb;
      if (p.vec_ok && cnt == kSeg) {
        uint4* o = reinterpret_cast<uint4*>(dst);
        o[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        o[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
      } else {
        for (int i = 0; i < cnt; ++i) dst[i] = (uint16_t)(wv[i / 2] >> (16 * (i & 1)));
      }
    }
    };

  for (int k = 0; k < nchunks; ++k) {
    const int64_t t0 = (int64_t)k * kT;
    const int tl = (int)min((int64_t)kT, L - t0);
    Raw<kN, kCH>& r = raw[k & 1];
    cp_async_wait_all();
    __syncthreads();  // raw bytes of chunk k landed; the scan of chunk k - 1 is complete
    if (k > 0) store_chunk(k - 1);  // reads sY and the raw bytes of chunk k - 1 only

    // ---- stage: (delta, delta x) per (c, t); B, C dequantised to [t][n]
    for (int w = tid; w < kCH * SEGS; w += NT) {
      const int c = w / SEGS, tb = (w % SEGS) * kSeg;
      float xs = 1.0f, bias = 0.0f;
      if (c < nc) {
        const int64_t ch = c0 + c;
        if (kXFmt == SSMQ_X_INT8_GROUP) {
          const int xg = __ldg(p.x_group + ch);
          if ((unsigned)xg < (unsigned)p.n_x_groups) {
            xs = __ldg(p.x_scale + xg);
          } else {
            xs = 0.0f;
            flags |= SSMQ_DEV_BAD_GROUP;
          }
        }
        bias = p.dt_bias ? __ldg(p.dt_bias + ch) : 0.0f;
      }
      const uint4 xw = *reinterpret_cast<const uint4*>(&r.x[c][tb]);
      const uint32_t xb[4] = {xw.x, xw.y, xw.z, xw.w};
      const uint4 d0 = *reinterpret_cast<const uint4*>(&r.dt[c][tb]);
      const uint4 d1 = *reinterpret_cast<const uint4*>(&r.dt[c][tb + 8]);
      const uint32_t dw[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
      float4 out[kSeg / 2];
#pragma unroll
      for (int i = 0; i < kSeg; i += 2) {
        float dd[2], dx[2];
        const float2 dtf = __half22float2(*reinterpret_cast<const __half2*>(&dw[i >> 1]));
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = i + e;
          const uint32_t code = (xb[t >> 2] >> (8 * (t & 3))) & 0xFFu;
          const float xv = kXFmt == SSMQ_X_INT8_GROUP ? s8_to_f32(xb[t >> 2] ^ 0x80808080u, t & 3) * xs
                                                      : se_decode(code, p.se);
          const float dv = (e ? dtf.y : dtf.x) + bias;
          float delta = p.softplus ? softplus_f(dv) : dv;
          if (c >= nc || tb + t >= tl) delta = 0.0f;
          dd[e] = delta;
          dx[e] = delta * xv;
        }
        out[i / 2] = make_float4(dd[0], dx[0], dd[1], dx[1]);
      }
      float4* dst = reinterpret_cast<float4*>(&sDD[c][tb]);
#pragma unroll
      for (int i = 0; i < kSeg / 2; ++i) dst[i] = out[i];
    }
    for (int w = tid; w < 2 * kN * SEGS; w += NT) {
      const int which = w / (kN * SEGS), rem = w % (kN * SEGS);
      const int n = rem % kN, tb = (rem / kN) * kSeg;
      const float sc = __ldg((which ? p.C_scale : p.B_scale) + g * spg + n / p.gs);
      const uint4 qw = *reinterpret_cast<const uint4*>(which ? &r.C[n][tb] : &r.B[n][tb]);
      const uint32_t qb[4] = {qw.x ^ 0x80808080u, qw.y ^ 0x80808080u, qw.z ^ 0x80808080u,
                              qw.w ^ 0x80808080u};
      float* dst = which ? &sC[0][0] : &sB[0][0];
#pragma unroll
      for (int i = 0; i < kSeg; ++i) {
        const float v = s8_to_f32(qb[i >> 2], i & 3) * sc;
        dst[(tb + i) * kN + n] = tb + i < tl ? v : 0.0f;
      }
    }
    __syncthreads();

    // ---- prefetch the next chunk (into the buffer chunk k - 1 used) while
    // this one is scanned
    if (k + 1 < nchunks)
      fetch_chunk<kN, kCH>(p, raw[(k + 1) & 1], bb, g, c0, nc, t0 + kT,
                           (int)min((int64_t)kT, L - t0 - kT), tid, NT);
    cp_async_commit();

    // ---- scan
#pragma unroll 2
    for (int tg = 0; tg < kT / LPC; ++tg) {
      float part[LPC];
#pragma unroll
      for (int kk = 0; kk < LPC; ++kk) {
        const int t = tg * LPC + kk;
        const float2 dd = sDD[lc][t];
        float2 bq[NP], cq[NP];
        if (kSPL == 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(&sB[t][lj * kSPL]);
          const float4 c4 = *reinterpret_cast<const float4*>(&sC[t][lj * kSPL]);
          bq[0] = make_float2(b4.x, b4.y);
          bq[NP - 1] = make_float2(b4.z, b4.w);
          cq[0] = make_float2(c4.x, c4.y);
          cq[NP - 1] = make_float2(c4.z, c4.w);
        } else {
          bq[0] = *reinterpret_cast<const float2*>(&sB[t][lj * kSPL]);
          cq[0] = *reinterpret_cast<const float2*>(&sC[t][lj * kSPL]);
        }
        const float2 dl = make_float2(dd.x, dd.x), dxv = make_float2(dd.y, dd.y);
        float2 q = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          const float2 r = fmul2(dl, ap[i]);
          const float2 e = make_float2(ex2_sfu(r.x), ex2_sfu(r.y));
          hp[i] = ffma2(e, hp[i], fmul2(dxv, bq[i]));
          q = i == 0 ? fmul2(cq[i], hp[i]) : ffma2(cq[i], hp[i], q);
        }
        part[kk] = q.x + q.y;
      }
      sY[lc][tg * LPC + lj] = reduce_scatter<LPC>(part, lj);
    }
  }
  __syncthreads();
  store_chunk(nchunks - 1);

  if (lvalid && p.h_final)
#pragma unroll
    for (int i = 0; i < NP; ++i)
      *reinterpret_cast<float2*>(p.h_final + (bb * d + lch) * kN + lj * kSPL + 2 * i) = hp[i];
  flag_status(p.status, flags);
}

template <int kN, int kCH, int kSPL>
cudaError_t launch_m1(const M1Params& prm, int xfmt, int64_t batch, cudaStream_t st) {
  M1Params p = prm;
  const int dg = (int)(p.d / p.G);
  p.n_ctile = (dg + kCH - 1) / kCH;
  const dim3 grid((unsigned)(p.n_ctile * p.G), (unsigned)batch);
  const dim3 block(kCH * (kN / kSPL));
  const size_t smem = sizeof(M1Smem<kN, kCH>);
  auto kern = xfmt == SSMQ_X_SOFTEDGE ? m1_scan_kernel<kN, kCH, kSPL, SSMQ_X_SOFTEDGE>
                                      : m1_scan_kernel<kN, kCH, kSPL, SSMQ_X_INT8_GROUP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, block, smem, st>>>(p);
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
    case 4: return launch_m1<4, 32, 4>(p, a.x_format, a.batch, st);
    case 8: return launch_m1<8, 16, 4>(p, a.x_format, a.batch, st);
    case 16: return launch_m1<16, 16, 4>(p, a.x_format, a.batch, st);
    case 32: return launch_m1<32, 16, 4>(p, a.x_format, a.batch, st);
    case 64: return launch_m1<64, 8, 4>(p, a.x_format, a.batch, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ssmq
