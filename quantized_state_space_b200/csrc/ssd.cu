// Mamba-2 SSD chunked scan on W8A8 operands, sm_100a tensor cores (tcgen05).
//
// SSDi8 (arxivdaily card), abstract: Mamba-2's structured state-space duality
// runs a recurrent mode and an attention mode, and the element-wise products
// can be kept apart from the matrix products.  Quamba2 abstract: 8-bit x per
// clustered channel group, 8-bit B / C per state group.  Per head h (scalar
// A_h, state P x N) and tile of Q = 128 steps with S_t = sum_{r<=t} delta_r A_h:
//   CB        = C B^T                                        (MMA0, K = N)
//   M[t,s]    = CB[t,s] exp(S_t - S_s) delta_s,  s <= t       (CUDA cores)
//   Y_diag    = M X                                          (MMA1, K = Q)
//   Y_off     = C h_prev^T, row t scaled by exp(S_t)          (MMA2, K = N)
//   y         = Y_diag + Y_off + D x   (times silu(z))
//   h_next    = exp(S_last) h_prev + B^T (w X),
//               w_s = exp(S_last - S_s) delta_s               (MMA3, K = Q)
// The element-wise decay products stay on the CUDA cores in fp32; the tensor
// cores only see exact int8 values (as binary16) or power-of-two-normalised
// binary16 operands:
//   - C and B are int8 codes (exact); the per-state-group scales enter as
//     w'_n = sC_n sB_n / max_n(sC sB) on C (one rounding, range <= 127);
//   - each row of M is scaled by a power of two so its largest entry lies in
//     [2^14, 2^15) (undone in fp32 after the MMA);
//   - the state operand of MMA2 and the w X operand of MMA3 are split into a
//     binary16 high part and a binary16 residual (two MMAs each), with a
//     tile-wide power-of-two normalisation: the state then carries ~22 bits.
// One CTA (8 warps) owns one (batch, head) and walks the sequence in tiles;
// the fp32 state lives in registers (row n, 32 of the 64 p per thread),
// accumulators in TMEM (256 columns), operands in shared memory (176 KB).
// The chunk length of the interface only fixes where the decomposition
// restarts; the result is the recurrence's for any length, so the kernel uses
// 128-step tiles for every accepted chunk length.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace ssmq {
namespace {

constexpr int kQ = 128;  // tile length
constexpr int kP = 64;   // head dim
constexpr int kN = 128;  // state dim
constexpr int kThreads = 256;
constexpr uint32_t kWaitLimit = 1u << 22;  // mbarrier polls before giving up
constexpr uint32_t kTmemCols = 256;

// shared-memory map (bytes)
constexpr int OFF_C = 0;                        // C codes * w'     [t][n]  K-major   32 KB
constexpr int OFF_B = OFF_C + kQ * kN * 2;      // B codes          [s][n]            32 KB
constexpr int OFF_X = OFF_B + kQ * kN * 2;      // x (exact)        [s][p]  MN-major  16 KB
constexpr int OFF_XH = OFF_X + kQ * kP * 2;     // w x hi           [s][p]            16 KB
constexpr int OFF_XL = OFF_XH + kQ * kP * 2;    // w x lo                             16 KB
constexpr int OFF_HH = OFF_XL + kQ * kP * 2;    // state hi         [n][p]  MN-major  16 KB
constexpr int OFF_HL = OFF_HH + kN * kP * 2;    // state lo                           16 KB
constexpr int OFF_M = OFF_HL + kN * kP * 2;     // M                [t][s]  K-major   32 KB
constexpr int OFF_F = OFF_M + kQ * kQ * 2;      // fp32 scalars
// fp32 scalar arrays (in floats, from OFF_F)
constexpr int F_S2 = 0;            // S_t * log2(e)            [128]
constexpr int F_DW = F_S2 + kQ;    // delta_s                  [128]
constexpr int F_WX = F_DW + kQ;    // w_s = exp(S_last-S_s) d_s [128]
constexpr int F_ES = F_WX + kQ;    // exp(S_t)                 [128]
constexpr int F_RS = F_ES + kQ;    // 2^e_t row scale of M     [128]
constexpr int F_RM = F_RS + kQ;    // row max halves           [2][128]
constexpr int F_WN = F_RM + 2 * kQ;  // w'_n                   [128]
constexpr int F_SB = F_WN + kN;    // sB_n                     [128]
constexpr int F_SX = F_SB + kN;    // x scale per p            [64]
constexpr int F_RED = F_SX + kP;   // reductions               [32]
constexpr int F_END = F_RED + 32;
constexpr int kSmemBytes = OFF_F + F_END * 4;

struct SsdParams {
  int64_t L, H, G;
  int gs;
  int xfmt;
  const void* x;
  const int32_t* x_group;
  const float* x_scale;
  int n_x_groups;
  SeSteps se;
  int se_shift;   // log2 ratio
  float x_bound;  // largest |x_exact| a code can produce
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
};

// 2^e as an exact float for |e| < 126
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// exponent e so that a * 2^-e lies in [2^14, 2^15) (0 for a == 0 / non-finite)
__device__ __forceinline__ int norm_exp(float a) {
  if (!(a > 0.0f) || !isfinite(a)) return 0;
  int E;
  frexpf(a, &E);  // a = m 2^E, m in [0.5, 1)
  return max(-100, min(100, E - 15));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  return (uint32_t)__half_as_ushort(__float2half_rn(a)) |
         ((uint32_t)__half_as_ushort(__float2half_rn(b)) << 16);
}

// value of one x element as an exactly representable binary16 number, the
// column scale being applied after the MMA
__device__ __forceinline__ float x_exact(uint32_t code, int xfmt, int shift) {
  if (xfmt == SSMQ_X_SOFTEDGE) {
    int q, mode;
    se_split(code, q, mode);
    return mode == 0 ? (float)q : (mode == 1 ? (float)q * pow2i(-shift) : (float)q * pow2i(shift));
  }
  return (float)(int8_t)(code & 0xFFu);
}

__device__ __forceinline__ float block_max(float v, float* red, int tid) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

__global__ void __launch_bounds__(kThreads, 1) ssd_kernel(const SsdParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  float* F = reinterpret_cast<float*>(smem + OFF_F);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t u = blockIdx.x;  // b * H + h
  const int64_t H = p.H, L = p.L;
  const int64_t bb = u / H, hd = u % H;
  const int64_t g = hd * p.G / H;
  const int row = 32 * (warp & 3) + lane;  // TMEM lane owned by this thread
  const int half = warp >> 2;              // column half
  const uint32_t s_base = tc::smem_u32(smem);
  uint32_t flags = 0;

  // ---- per-CTA constants
  if (tid < kN) {
    const int si = (int)g * (kN / p.gs) + tid / p.gs;
    const float sc = __ldg(p.C_scale + si), sb = __ldg(p.B_scale + si);
    F[F_WN + tid] = sc * sb;
    F[F_SB + tid] = sb;
  }
  if (tid < kP) {
    float sx = p.se.s[0];
    if (p.xfmt == SSMQ_X_INT8_GROUP) {
      const int xg = __ldg(p.x_group + hd * kP + tid);
      if ((unsigned)xg < (unsigned)p.n_x_groups) {
        sx = __ldg(p.x_scale + xg);
      } else {
        sx = 0.0f;
        flags |= SSMQ_DEV_BAD_GROUP;
      }
    }
    F[F_SX + tid] = sx;
  }
  if (tid == 0) abort_flag = 0;
  if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&bars[0], 1);
    tc::mbar_init(&bars[1], 1);
  }
  __syncthreads();
  const float wmax = block_max(tid < kN ? F[F_WN + tid] : 0.0f, F + F_RED, tid);
  if (tid < kN) F[F_WN + tid] = wmax > 0.0f ? F[F_WN + tid] / wmax : 0.0f;
  const float A2 = __ldg(p.A + hd) * kLog2e;
  const float bias = p.dt_bias ? __ldg(p.dt_bias + hd) : 0.0f;
  const float Dh = p.D ? __ldg(p.D + hd) : 0.0f;

  // ---- initial state: thread (row = n, half) holds p in [32 half, 32 half + 32)
  float hs[32];
  {
    float* stage = reinterpret_cast<float*>(smem + OFF_M);  // P x N fp32 = 32 KB
    if (p.h0) {
      const float4* src = reinterpret_cast<const float4*>(p.h0 + u * kP * kN);
      for (int i = tid; i < kP * kN / 4; i += kThreads) reinterpret_cast<float4*>(stage)[i] = src[i];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 32; ++j) hs[j] = p.h0 ? stage[(32 * half + j) * kN + row] : 0.0f;
    __syncthreads();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
  const uint32_t T_CB = 0, T_ACC = 0, T_YD = 128, T_YO = 192;

  uint32_t phase = 0;
  for (int64_t t0 = 0; t0 < L; t0 += kQ, phase ^= 1u) {
    const int ql = (int)min((int64_t)kQ, L - t0);
    // ---- delta, S = cumsum(delta A) (threads 0..127, one step each)
    if (tid < kQ) {
      float dl = 0.0f;
      if (tid < ql) {
        const float v = h2f(p.dt[(bb * L + t0 + tid) * H + hd]) + bias;
        dl = p.softplus ? softplus_f(v) : v;
      }
      float s = dl * A2;  // log2 units
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += n;
      }
      if (lane == 31) F[F_RED + warp] = s;  // warp totals (warps 0..3)
      F[F_DW + tid] = dl;
      F[F_S2 + tid] = s;
    }
    __syncthreads();
    if (tid < kQ) {
      float off = 0.0f;
      for (int w = 0; w < (tid >> 5); ++w) off += F[F_RED + w];
      F[F_S2 + tid] += off;
    }
    __syncthreads();
    const float s_last = F[F_S2 + kQ - 1];
    float wx = 0.0f;
    if (tid < kQ) {
      const float s2 = F[F_S2 + tid];
      wx = ex2_sfu(s_last - s2) * F[F_DW + tid];
      F[F_WX + tid] = wx;
      F[F_ES + tid] = ex2_sfu(s2);
    }
    const float wx_max = block_max(wx, F + F_RED, tid);
    const int ex = norm_exp(wx_max * p.x_bound);  // x_bound >= max |x_exact|
    const float xsc = pow2i(-ex);

    // ---- stage C (codes * w'_n) and B (codes) rows: thread -> (row, 64 states)
    {
      const int r = tid >> 1, part = tid & 1;
      const bool ok = r < ql;
      const int64_t ro = ((bb * L + t0 + r) * p.G + g) * kN + 64 * part;
      uint4 cq[4], bq[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        cq[i] = ok ? __ldg(reinterpret_cast<const uint4*>(p.C + ro) + i) : make_uint4(0, 0, 0, 0);
        bq[i] = ok ? __ldg(reinterpret_cast<const uint4*>(p.B + ro) + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t cw[4] = {cq[i].x, cq[i].y, cq[i].z, cq[i].w};
        const uint32_t bw[4] = {bq[i].x, bq[i].y, bq[i].z, bq[i].w};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // 8 states per 16-byte core-matrix row
          const int n0 = 64 * part + 16 * i + 8 * hh;
          uint32_t oc[4], ob[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t wc = cw[2 * hh + k / 2], wb = bw[2 * hh + k / 2];
            const int sh = 16 * (k & 1);
            const float c0 = (float)(int8_t)(wc >> sh), c1 = (float)(int8_t)(wc >> (sh + 8));
            const float b0 = (float)(int8_t)(wb >> sh), b1 = (float)(int8_t)(wb >> (sh + 8));
            oc[k] = pack_h2(c0 * F[F_WN + n0 + 2 * k], c1 * F[F_WN + n0 + 2 * k + 1]);
            ob[k] = pack_h2(b0, b1);
          }
          *reinterpret_cast<uint4*>(smem + OFF_C + tc::kmaj_off(r, n0, kN)) =
              make_uint4(oc[0], oc[1], oc[2], oc[3]);
          *reinterpret_cast<uint4*>(smem + OFF_B + tc::kmaj_off(r, n0, kN)) =
              make_uint4(ob[0], ob[1], ob[2], ob[3]);
        }
      }
    }
    // ---- stage x (exact) and w x (hi / lo) rows: thread -> (row s, 32 p)
    {
      const int s = tid >> 1, part = tid & 1;
      const bool ok = s < ql;
      const int64_t xo = ((bb * L + t0 + s) * H + hd) * kP + 32 * part;
      uint4 xq[2];
#pragma unroll
      for (int i = 0; i < 2; ++i)
        xq[i] = ok ? __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.x) + xo) + i)
                   : make_uint4(0, 0, 0, 0);
      const float ws = F[F_WX + s] * xsc;
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {  // 8 p per group
        const uint4 q = xq[grp / 2];
        const uint32_t w0 = (grp & 1) ? q.z : q.x, w1 = (grp & 1) ? q.w : q.y;
        float xv[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          xv[k] = x_exact((w0 >> (8 * k)) & 0xFFu, p.xfmt, p.se_shift);
          xv[4 + k] = x_exact((w1 >> (8 * k)) & 0xFFu, p.xfmt, p.se_shift);
        }
        uint32_t ox[4], oh[4], ol[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          ox[k] = pack_h2(xv[2 * k], xv[2 * k + 1]);
          const float v0 = ws * xv[2 * k], v1 = ws * xv[2 * k + 1];
          const __half h0v = __float2half_rn(v0), h1v = __float2half_rn(v1);
          oh[k] = (uint32_t)__half_as_ushort(h0v) | ((uint32_t)__half_as_ushort(h1v) << 16);
          ol[k] = pack_h2(v0 - __half2float(h0v), v1 - __half2float(h1v));
        }
        const uint32_t off = tc::mnmaj_off(32 * part + 8 * grp, s, kP);
        *reinterpret_cast<uint4*>(smem + OFF_X + off) = make_uint4(ox[0], ox[1], ox[2], ox[3]);
        *reinterpret_cast<uint4*>(smem + OFF_XH + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
        *reinterpret_cast<uint4*>(smem + OFF_XL + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
      }
    }
    // ---- stage the state (hi / lo) for Y_off: h'' = h w_max / sB_n, normalised
    float hmax = 0.0f;
    {
      const float f = F[F_SB + row] > 0.0f ? wmax / F[F_SB + row] : 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) hmax = fmaxf(hmax, fabsf(hs[j] * f));
    }
    const float hmax_all = block_max(hmax, F + F_RED, tid);
    const int eh = norm_exp(hmax_all);
    {
      const float f = (F[F_SB + row] > 0.0f ? wmax / F[F_SB + row] : 0.0f) * pow2i(-eh);
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        uint32_t oh[4], ol[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float v0 = hs[8 * grp + 2 * k] * f, v1 = hs[8 * grp + 2 * k + 1] * f;
          const __half h0v = __float2half_rn(v0), h1v = __float2half_rn(v1);
          oh[k] = (uint32_t)__half_as_ushort(h0v) | ((uint32_t)__half_as_ushort(h1v) << 16);
          ol[k] = pack_h2(v0 - __half2float(h0v), v1 - __half2float(h1v));
        }
        const uint32_t off = tc::mnmaj_off(32 * half + 8 * grp, row, kP);
        *reinterpret_cast<uint4*>(smem + OFF_HH + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
        *reinterpret_cast<uint4*>(smem + OFF_HL + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
      }
    }
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();

    // ---- MMA0: CB = C' B^T  (M = t, N = s, K = n)
    if (tid == 0) {
      tc::fence_after();
      const uint32_t id = tc::idesc_f16(kQ, kQ, false, false);
#pragma unroll
      for (int k0 = 0; k0 < kN; k0 += 16)
        tc::mma_f16(tmem + T_CB, tc::kmaj_desc(s_base + OFF_C, k0, kN),
                    tc::kmaj_desc(s_base + OFF_B, k0, kN), id, k0 > 0);
      tc::mma_commit(&bars[0]);
    }
    __syncwarp();
    if (!tc::mbar_wait(&bars[0], phase, kWaitLimit)) {
      flags |= SSMQ_DEV_TIMEOUT;
      atomicExch(&abort_flag, 1);
    }
    if (__syncthreads_or(abort_flag)) break;
    tc::fence_after();

    // ---- M = CB * exp(S_t - S_s) * delta_s * w_max, row-normalised, s <= t
    {
      const int t = row;
      const float st = F[F_S2 + t];
      float mv[64];
      float rmax = 0.0f;
      const bool any = (64 * half) <= t;  // columns of this half reach the diagonal
      if (any) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[32];
          tc::tmem_ld32(tmem + t_lane + T_CB + 64 * half + 32 * c, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s = 64 * half + 32 * c + j;
            const float m = s <= t ? v[j] * ex2_sfu(st - F[F_S2 + s]) * F[F_DW + s] * wmax : 0.0f;
            mv[32 * c + j] = m;
            rmax = fmaxf(rmax, fabsf(m));
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) mv[j] = 0.0f;
      }
      F[F_RM + half * kQ + t] = rmax;
      __syncthreads();
      const int et = norm_exp(fmaxf(F[F_RM + t], F[F_RM + kQ + t]));
      const float sc = pow2i(-et);
      if (half == 0) F[F_RS + t] = pow2i(et);
#pragma unroll
      for (int grp = 0; grp < 8; ++grp) {
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = pack_h2(mv[8 * grp + 2 * k] * sc, mv[8 * grp + 2 * k + 1] * sc);
        *reinterpret_cast<uint4*>(smem + OFF_M + tc::kmaj_off(t, 64 * half + 8 * grp, kQ)) =
            make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();

    // ---- MMA1 (Y_diag), MMA2 (Y_off, hi + lo), MMA3 (state, hi + lo)
    if (tid == 0) {
      tc::fence_after();
      const uint32_t id_y = tc::idesc_f16(kQ, kP, false, true);
      const uint32_t id_s = tc::idesc_f16(kN, kP, true, true);
#pragma unroll
      for (int k0 = 0; k0 < kQ; k0 += 16)
        tc::mma_f16(tmem + T_YD, tc::kmaj_desc(s_base + OFF_M, k0, kQ),
                    tc::mnmaj_desc(s_base + OFF_X, k0, kP), id_y, k0 > 0);
#pragma unroll
      for (int k0 = 0; k0 < kN; k0 += 16)
        tc::mma_f16(tmem + T_YO, tc::kmaj_desc(s_base + OFF_C, k0, kN),
                    tc::mnmaj_desc(s_base + OFF_HH, k0, kP), id_y, k0 > 0);
#pragma unroll
      for (int k0 = 0; k0 < kN; k0 += 16)
        tc::mma_f16(tmem + T_YO, tc::kmaj_desc(s_base + OFF_C, k0, kN),
                    tc::mnmaj_desc(s_base + OFF_HL, k0, kP), id_y, 1u);
#pragma unroll
      for (int k0 = 0; k0 < kQ; k0 += 16)
        tc::mma_f16(tmem + T_ACC, tc::mnmaj_desc(s_base + OFF_B, k0, kN),
                    tc::mnmaj_desc(s_base + OFF_XH, k0, kP), id_s, k0 > 0);
#pragma unroll
      for (int k0 = 0; k0 < kQ; k0 += 16)
        tc::mma_f16(tmem + T_ACC, tc::mnmaj_desc(s_base + OFF_B, k0, kN),
                    tc::mnmaj_desc(s_base + OFF_XL, k0, kP), id_s, 1u);
      tc::mma_commit(&bars[1]);
    }
    __syncwarp();
    if (!tc::mbar_wait(&bars[1], phase, kWaitLimit)) {
      flags |= SSMQ_DEV_TIMEOUT;
      atomicExch(&abort_flag, 1);
    }
    if (__syncthreads_or(abort_flag)) break;
    tc::fence_after();

    // ---- y = Y_diag 2^e_t sx + exp(S_t) 2^e_h Y_off + D x  (thread: row t, 32 p)
    {
      const int t = row;
      float yd[32], yo[32];
      tc::tmem_ld32(tmem + t_lane + T_YD + 32 * half, yd);
      tc::tmem_ld32(tmem + t_lane + T_YO + 32 * half, yo);
      if (t < ql) {
        const float rs = F[F_RS + t], es = F[F_ES + t] * pow2i(eh);
        const int64_t yo_off = ((bb * L + t0 + t) * H + hd) * kP + 32 * half;
        const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.x) + yo_off);
        const uint4 xa = __ldg(xr), xb = __ldg(xr + 1);
        const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        uint32_t zw[16];
        if (p.z) {
          const uint4* zr = reinterpret_cast<const uint4*>(p.z + yo_off);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 zz = __ldg(zr + i);
            zw[4 * i] = zz.x;
            zw[4 * i + 1] = zz.y;
            zw[4 * i + 2] = zz.z;
            zw[4 * i + 3] = zz.w;
          }
        }
        uint32_t out[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float r2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int pj = j + e;
            const float sx = F[F_SX + 32 * half + pj];
            const float xv = x_exact((xw[pj >> 2] >> (8 * (pj & 3))) & 0xFFu, p.xfmt, p.se_shift) * sx;
            float yv = yd[pj] * rs * sx + es * yo[pj] + Dh * xv;
            if (p.z) yv *= silu_f(h2f((uint16_t)(zw[pj >> 1] >> (16 * (pj & 1)))));
            r2[e] = yv;
          }
          out[j / 2] = (uint32_t)f2h(r2[0]) | ((uint32_t)f2h(r2[1]) << 16);
        }
        uint4* yr = reinterpret_cast<uint4*>(p.y + yo_off);
#pragma unroll
        for (int i = 0; i < 4; ++i) yr[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
      }
    }
    // ---- state: h = exp(S_last) h + sB_n sx_p 2^-e_x acc  (thread: row n, 32 p)
    {
      float acc[32];
      tc::tmem_ld32(tmem + t_lane + T_ACC + 32 * half, acc);
      const float decay = ex2_sfu(s_last);
      const float f = F[F_SB + row] * pow2i(ex);
#pragma unroll
      for (int j = 0; j < 32; ++j) hs[j] = fmaf(decay, hs[j], f * F[F_SX + 32 * half + j] * acc[j]);
    }
    tc::fence_before();
    __syncthreads();
  }

  // ---- final state (P, N) through shared memory for coalesced stores
  if (p.h_final) {
    float* stage = reinterpret_cast<float*>(smem + OFF_M);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 32; ++j) stage[(32 * half + j) * kN + row] = hs[j];
    __syncthreads();
    float4* dst = reinterpret_cast<float4*>(p.h_final + u * kP * kN);
    for (int i = tid; i < kP * kN / 4; i += kThreads) dst[i] = reinterpret_cast<float4*>(stage)[i];
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
  flag_status(p.status, flags);
}

}  // namespace

size_t ssd_workspace_bytes(const ssmq_ssd_args&) { return 0; }

cudaError_t launch_ssd(const ssmq_ssd_args& a, void*, cudaStream_t st) {
  const int64_t units = a.batch * a.nheads;
  if (units == 0) return cudaSuccess;
  if (a.seqlen == 0) {
    if (!a.h_final) return cudaSuccess;
    const size_t bytes = sizeof(float) * (size_t)(units * a.headdim * a.dstate);
    return a.h0 ? cudaMemcpyAsync(a.h_final, a.h0, bytes, cudaMemcpyDeviceToDevice, st)
                : cudaMemsetAsync(a.h_final, 0, bytes, st);
  }
  SsdParams p{};
  p.L = a.seqlen;
  p.H = a.nheads;
  p.G = a.ngroups;
  p.gs = a.state_group_size;
  p.xfmt = a.x_format;
  p.x = a.x;
  p.x_group = a.x_group;
  p.x_scale = a.x_scale;
  p.n_x_groups = a.n_x_groups;
  p.se = se_steps(a.x_format == SSMQ_X_SOFTEDGE ? a.se_scale : 1.0f, a.se_log2_ratio);
  p.se_shift = a.se_log2_ratio;
  p.x_bound = a.x_format == SSMQ_X_SOFTEDGE ? fmaxf(63.0f, 31.0f * (float)(1 << a.se_log2_ratio))
                                            : 128.0f;
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
  cudaError_t e = cudaFuncSetAttribute(ssd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  ssd_kernel<<<(unsigned)units, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace ssmq
