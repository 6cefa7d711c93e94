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
//     w'_n = fl16(sC_n sB_n / max_n(sC sB)) on C (C' = fl16(c w'_n), one
//     packed half2 multiply); the state operand of MMA2 carries sC_n / w'_n
//     so the rounding of w' cancels there;
//   - each row of M is scaled by a power of two so its largest entry lies in
//     [2^14, 2^15) (undone in fp32 after the MMA);
//   - the w X operand of MMA3 is split into a binary16 high part and a
//     binary16 residual (two MMAs), with a tile-wide power-of-two
//     normalisation, so the state increments carry ~22 bits; the state
//     operand of MMA2 (which only feeds y) is one normalised binary16 value.
// The head-independent operands (C' and B of a tile) are written once per
// (batch, group) by ssd_operand_kernel into the workspace, in the layouts the
// MMAs read, and bulk-copied into shared memory by each head's CTA.
// One CTA (16 warps) owns one (batch, head) and walks the sequence in tiles;
// warp 0 prepares the next tile's decay factors while the others finish the
// current tile's outputs;
// the fp32 state lives in registers (row n, 16 of the 64 p per thread: warp w
// reads TMEM lanes 32 (w % 4).. and columns 16 (w / 4)..), accumulators in
// TMEM (512 columns), operands in shared memory (183 KB, including the raw
// int8 x rows of the next tile, prefetched with cp.async during this one).
// The chunk length of the interface only fixes where the decomposition
// restarts; the result is the recurrence's for any length, so the kernel uses
// 128-step tiles for every accepted chunk length.
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "stream.cuh"
#include "tc.cuh"

namespace ssmq {
namespace {

constexpr int kQ = 128;  // tile length
constexpr int kP = 64;   // head dim
constexpr int kN = 128;  // state dim
constexpr int kThreads = 512;
constexpr uint32_t kWaitLimit = 1u << 20;  // mbarrier probes (~1 us each) before giving up
constexpr uint32_t kTmemCols = 512;
constexpr int kIssueWarp = 14;   // rb 2, q4 3: an all-zero block of M
constexpr int kFactorWarp = 9;   // rb 1, q4 2: an all-zero block of M

// shared-memory map (bytes)
// two operand buffers (tiles alternate): C' codes * w' [t][n] K-major, then
// B codes [s][n] K-major, 32 KB each
constexpr int OFF_OPS = 0;
constexpr int OFF_X = OFF_OPS + 4 * kQ * kN * 2;  // x (exact)      [s][p]  MN-major  16 KB
constexpr int OFF_XH = OFF_X + kQ * kP * 2;     // w x hi           [s][p]            16 KB
constexpr int OFF_XL = OFF_XH + kQ * kP * 2;    // w x lo                             16 KB
constexpr int OFF_HH = OFF_XL + kQ * kP * 2;    // state            [n][p]  MN-major  16 KB
constexpr int OFF_F = OFF_HH + kN * kP * 2;    // fp32 scalars
// the initial and final states (P x N fp32, 32 KB) pass through OFF_X..OFF_HH
constexpr int OFF_STATE = OFF_X;
// fp32 scalar arrays (in floats, from OFF_F).  The per-step arrays of a tile
// are double-buffered: warp 0 fills the next tile's while the others finish
// this one.
constexpr int F_S2 = 0;                 // S_t * log2(e)                       [2][128]
constexpr int F_DW = F_S2 + 2 * kQ;     // delta_s                             [2][128]
constexpr int F_WX = F_DW + 2 * kQ;     // w_s = exp(S_last - S_s) delta_s      [2][128]
constexpr int F_ES = F_WX + 2 * kQ;     // exp(S_t)                            [2][128]
constexpr int F_CW = F_ES + 2 * kQ;     // exp(S_p(s) - S_s) d_s w_max, p(s) = s | 31  [2][128]
constexpr int F_CD = F_CW + 2 * kQ;     // exp(S_m(s) - S_s) d_s w_max, m(s) = s & ~31  [2][128]
constexpr int F_BS = F_CD + 2 * kQ;     // spread max - min of S (log2) per 32-step block  [2][4]
constexpr int F_RS = F_BS + 8;          // 2^e_t row scale of M                [128]
constexpr int F_RM = F_RS + kQ;         // row max quarters                    [4][128]
constexpr int F_WH = F_RM + 4 * kQ;     // w'_n as binary16 pairs              [64]
constexpr int F_HF = F_WH + kN / 2;     // sC_n / w'_n (state operand factor)  [128]
constexpr int F_SB = F_HF + kN;         // sB_n                                [128]
constexpr int F_SX = F_SB + kN;         // x scale per p                       [64]
constexpr int F_YS = F_SX + kP;         // int8-y scale per p                  [64]
constexpr int F_YR = F_YS + kP;         // its reciprocal (0: exact division)  [64]
constexpr int F_YOK = F_YR + kP;        // 1 if the p's output cluster id is valid  [64]
constexpr int F_RED = F_YOK + kP;       // reductions: w max, S_last, per-warp state max  [32]
constexpr int F_END = F_RED + 32;
// raw int8 rows of the next tile, fetched with cp.async during this tile
constexpr int OFF_RAW = (OFF_F + F_END * 4 + 127) / 128 * 128;
constexpr int OFF_RX = OFF_RAW;                 // x codes [t][p]   8 KB
constexpr int kSmemBytes = OFF_RX + kQ * kP;
static_assert(kSmemBytes + 1024 <= 232448, "shared memory of one CTA");
// operand blocks written by ssd_operand_kernel, per (batch, group, tile):
// C' then B, each in the K-major canonical layout of an operand buffer
constexpr int kOpBlock = kQ * kN * 2;           // 32 KB
constexpr int kOpTile = 2 * kOpBlock;           // 64 KB

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
  int8_t* y_q;
  const int32_t* y_group;
  const float* y_scale;
  int n_y_groups;
  float* h_final;
  uint32_t* status;
  const uint8_t* ops;  // operand blocks (workspace)
  int64_t ntiles;
  // work items: units [0, full) are whole sequences; each later unit is cut
  // into kseg segments of seg_tiles tiles whose local final states and total
  // log2-decays go to seg_state / seg_dec (index (unit - full) * kseg + seg)
  int64_t full;
  int kseg, seg_tiles;
  float* seg_state;
  float* seg_dec;
  float* dec_final;       // (b, H) total log2 decay of each sequence, or null
  const float* h_carry;   // carry-in mode of the second kernel: (b, H, P, N)
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

__device__ __forceinline__ uint32_t pack_h2(float a, float b) { return pack_half2(a, b); }

// v = hi + lo with hi, lo binary16 (two packed pairs)
__device__ __forceinline__ void split_h2(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(v0, v1);
  const float2 hf = __half22float2(h);
  hi = h2_bits(h);
  lo = pack_half2(v0 - hf.x, v1 - hf.y);
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

// cp.async the x codes (P bytes per step) of the tile starting at t0 into the
// raw buffer; rows at or beyond ql are left as they are (the staging masks
// them).
__device__ __forceinline__ void fetch_tile(const SsdParams& p, uint8_t* smem, int64_t bb,
                                           int64_t hd, int64_t t0, int ql, int tid) {
  for (int w = tid; w < kQ * (kP / 16); w += kThreads) {
    const int r = w / (kP / 16), c = w % (kP / 16);
    if (r >= ql) continue;
    const int64_t xo = ((bb * p.L + t0 + r) * p.H + hd) * kP + 16 * c;
    tc::cp_async16(smem + OFF_RX + r * kP + 16 * (c ^ (r & 3)), static_cast<const uint8_t*>(p.x) + xo);
  }
  tc::cp_async_commit();
}

// w'_n = fl16(sC_n sB_n / max_n(sC sB)) of group g (every thread calls it;
// threads n < N return their w'_n, the others 0); wmax is returned too.
__device__ __forceinline__ __half group_wprime(const SsdParams& p, int64_t g, int tid, float* red,
                                               float& wmax, float& sc_n, float& sb_n) {
  sc_n = 0.0f;
  sb_n = 0.0f;
  if (tid < kN) {
    const int si = (int)g * (kN / p.gs) + tid / p.gs;
    sc_n = __ldg(p.C_scale + si);
    sb_n = __ldg(p.B_scale + si);
  }
  wmax = block_max(sc_n * sb_n, red, tid);
  return __float2half_rn(wmax > 0.0f ? sc_n * sb_n / wmax : 0.0f);
}

// The head-independent MMA operands of one (batch, group, tile): C' =
// fl16(codes * w'_n) and B (codes, exact) in the canonical K-major layouts the
// SSD kernel's MMAs read, written once for all heads of the group.  Rows at
// or beyond the sequence end are zero.
__global__ void __launch_bounds__(kThreads) ssd_operand_kernel(const SsdParams p, uint8_t* ops) {
  __shared__ float red[kThreads / 32];
  __shared__ __align__(16) __half wh[kN];
  const int tid = threadIdx.x;
  const int64_t tile = blockIdx.x, bg = blockIdx.y;
  const int64_t bb = bg / p.G, g = bg % p.G;
  float wmax, sc_n, sb_n;
  const __half w = group_wprime(p, g, tid, red, wmax, sc_n, sb_n);
  if (tid < kN) wh[tid] = w;
  __syncthreads();
  const int64_t t0 = tile * kQ;
  const int ql = (int)min((int64_t)kQ, p.L - t0);
  uint8_t* dst = ops + (bg * p.ntiles + tile) * kOpTile;
  // item (r, c): row r, states 16 c .. 16 c + 15; 8 consecutive items write
  // one 128-byte core matrix
  for (int it = tid; it < kQ * (kN / 16); it += kThreads) {
    const int c = it / kQ, r = it % kQ;
    uint4 cq = make_uint4(0, 0, 0, 0), bq = make_uint4(0, 0, 0, 0);
    if (r < ql) {
      const int64_t ro = ((bb * p.L + t0 + r) * p.G + g) * kN + 16 * c;
      cq = __ldg(reinterpret_cast<const uint4*>(p.C + ro));
      bq = __ldg(reinterpret_cast<const uint4*>(p.B + ro));
    }
    const uint32_t cw[4] = {cq.x ^ 0x80808080u, cq.y ^ 0x80808080u, cq.z ^ 0x80808080u,
                            cq.w ^ 0x80808080u};
    const uint32_t bw[4] = {bq.x ^ 0x80808080u, bq.y ^ 0x80808080u, bq.z ^ 0x80808080u,
                            bq.w ^ 0x80808080u};
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {  // 8 states per 16-byte core-matrix row
      const int n0 = 16 * c + 8 * hh;
      const uint4 wq = *reinterpret_cast<const uint4*>(wh + n0);
      const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
      uint32_t oc[4], ob[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t wc = cw[2 * hh + k / 2], wb = bw[2 * hh + k / 2];
        const int b0i = 2 * (k & 1);
        oc[k] = h2_bits(__hmul2(s8x2_to_h2(wc, b0i, b0i + 1),
                                *reinterpret_cast<const __half2*>(&wv[k])));
        ob[k] = h2_bits(s8x2_to_h2(wb, b0i, b0i + 1));
      }
      const uint32_t off = tc::kmaj_off(r, n0, kN);
      *reinterpret_cast<uint4*>(dst + off) = make_uint4(oc[0], oc[1], oc[2], oc[3]);
      *reinterpret_cast<uint4*>(dst + kOpBlock + off) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
  }
}

// Warp 0: delta, S = cumsum(delta A) (log2 units) and the per-step factors of
// the tile of ql steps whose dt values the lanes hold (4 steps per lane),
// into buffer fb; the tile's w max and S_last go to F_RED[0], F_RED[1].
// Warp 0: delta_t of the tile's steps 4 lane .. 4 lane + 3 (0 at or beyond
// ql) into dl, and S within the lane's steps (log2 units) into sc; off is the
// lane's offset (S = sc + off) and s_last S at the tile's last step.
__device__ __forceinline__ void tile_decay(int ql, const float (&dtv)[4], float bias,
                                           int softplus, float A2, int lane, float (&dl)[4],
                                           float (&sc)[4], float& off, float& s_last) {
  float run = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = 4 * lane + i;
    float d = 0.0f;
    if (t < ql) {
      const float v = dtv[i] + bias;
      d = softplus ? softplus_f(v) : v;
    }
    dl[i] = d;
    run += d * A2;
    sc[i] = run;
  }
  float ex = run;  // inclusive scan of the lane totals
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float n = __shfl_up_sync(0xffffffffu, ex, o);
    if (lane >= o) ex += n;
  }
  off = ex - run;
  s_last = __shfl_sync(0xffffffffu, ex, 31);
}

__device__ __forceinline__ void tile_factors(float* F, int fb, int ql, const float (&dtv)[4],
                                             float bias, int softplus, float A2, float wmax,
                                             int lane) {
  float dl[4], sc[4], off, s_last;
  tile_decay(ql, dtv, bias, softplus, A2, lane, dl, sc, off, s_last);
  float wmx = 0.0f;
  // S at the end and at the start of this lane's 32-step block (lanes 8 b + 7
  // and 8 b hold them), and the spread of S over the block
  const float s_blk = __shfl_sync(0xffffffffu, sc[3] + off, lane | 7);
  const float s_beg = __shfl_sync(0xffffffffu, sc[0] + off, lane & ~7);
  float smax = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])) + off;
  float smin = fminf(fminf(sc[0], sc[1]), fminf(sc[2], sc[3])) + off;
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) {
    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    smin = fminf(smin, __shfl_xor_sync(0xffffffffu, smin, o));
  }
  if ((lane & 7) == 0) F[F_BS + fb * 4 + (lane >> 3)] = smax - smin;
  float4 s2v, dwv, wxv, esv, cwv, cdv;
  float* o4[6] = {&s2v.x, &dwv.x, &wxv.x, &esv.x, &cwv.x, &cdv.x};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float s2 = sc[i] + off;
    const float w = ex2_sfu(s_last - s2) * dl[i];
    o4[0][i] = s2;
    o4[1][i] = dl[i];
    o4[2][i] = w;
    o4[3][i] = ex2_sfu(s2);
    o4[4][i] = ex2_sfu(s_blk - s2) * dl[i] * wmax;
    o4[5][i] = ex2_sfu(s_beg - s2) * dl[i] * wmax;
    wmx = fmaxf(wmx, w);
  }
  const int t0 = fb * kQ + 4 * lane;
  *reinterpret_cast<float4*>(F + F_S2 + t0) = s2v;
  *reinterpret_cast<float4*>(F + F_DW + t0) = dwv;
  *reinterpret_cast<float4*>(F + F_WX + t0) = wxv;
  *reinterpret_cast<float4*>(F + F_ES + t0) = esv;
  *reinterpret_cast<float4*>(F + F_CW + t0) = cwv;
  *reinterpret_cast<float4*>(F + F_CD + t0) = cdv;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) wmx = fmaxf(wmx, __shfl_xor_sync(0xffffffffu, wmx, o));
  if (lane == 0) {
    F[F_RED] = wmx;
    F[F_RED + 1] = s_last;
  }
}

template <bool kYQ>
__global__ void __launch_bounds__(kThreads, 1) ssd_kernel(const SsdParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(8) uint64_t bars[5];  // MMA0, MMA1, MMA2+3, operand buffers 0 / 1
  __shared__ int abort_flag;
  float* F = reinterpret_cast<float*>(smem + OFF_F);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // work item: a whole (batch, head) sequence, or segment seg of one
  int64_t u, t_beg = 0, t_end = p.L;
  int seg = 0, slot = -1;
  if ((int64_t)blockIdx.x < p.full) {
    u = blockIdx.x;  // b * H + h
  } else {
    const int64_t idx = (int64_t)blockIdx.x - p.full;
    u = p.full + idx / p.kseg;
    seg = (int)(idx % p.kseg);
    slot = (int)idx;
    t_beg = (int64_t)seg * p.seg_tiles * kQ;
    t_end = min(p.L, t_beg + (int64_t)p.seg_tiles * kQ);
  }
  const int64_t H = p.H, L = p.L;
  const int64_t bb = u / H, hd = u % H;
  const int64_t g = hd * p.G / H;
  const int row = 32 * (warp & 3) + lane;  // TMEM lane (row t or n) owned by this thread
  const int q4 = warp >> 2;                // column quarter
  const uint32_t s_base = tc::smem_u32(smem);
  uint32_t flags = 0;

  // ---- per-CTA constants
  float sc_n = 0.0f, sb_n = 0.0f;
  if (tid < kN) {
    const int si = (int)g * (kN / p.gs) + tid / p.gs;
    sc_n = __ldg(p.C_scale + si);
    sb_n = __ldg(p.B_scale + si);
    F[F_SB + tid] = sb_n;
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
    float ysc = 0.0f, yok = 1.0f;
    if (kYQ) {
      const int yg = __ldg(p.y_group + hd * kP + tid);
      if ((unsigned)yg < (unsigned)p.n_y_groups) {
        ysc = __ldg(p.y_scale + yg);
      } else {
        yok = 0.0f;
      }
    }
    const float yr = __frcp_rn(ysc);
    F[F_YS + tid] = ysc;
    F[F_YR + tid] = usable_recip(ysc, yr) ? yr : 0.0f;
    F[F_YOK + tid] = yok;
  }
  if (tid == 0) abort_flag = 0;
  if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&bars[0], 1);
    tc::mbar_init(&bars[1], 1);
    tc::mbar_init(&bars[2], 1);
    tc::mbar_init(&bars[3], 1);
    tc::mbar_init(&bars[4], 1);
  }
  __syncthreads();
  // The group's operand blocks of the work item's tile j (C' then B) go to
  // buffer j & 1 by one bulk copy, completion counted in bytes on
  // bars[3 + (j & 1)] (its (j >> 1)-th phase); tile j + 2 is fetched as soon
  // as tile j's MMAs are done.
  const uint8_t* ops_bg = p.ops + (bb * p.G + g) * p.ntiles * (int64_t)kOpTile;
  const int64_t n_tiles = (t_end - t_beg + kQ - 1) / kQ;
  uint32_t ops_n[2] = {0u, 0u};  // thread 0: copies issued per buffer
  auto issue_ops = [&](int64_t j) {
    stream::expect_tx(&bars[3 + (j & 1)], (uint32_t)kOpTile);
    stream::bulk_g2s(smem + OFF_OPS + (j & 1) * kOpTile, ops_bg + (t_beg / kQ + j) * kOpTile,
                     (uint32_t)kOpTile, &bars[3 + (j & 1)]);
    ++ops_n[j & 1];
  };
  auto ops_wait = [&](int64_t j) {
    return tc::mbar_wait(&bars[3 + (j & 1)], (uint32_t)(j >> 1) & 1u, kWaitLimit);
  };
  if (tid == 0) {
    issue_ops(0);
    if (n_tiles > 1) issue_ops(1);
  }
  const float wmax = block_max(sc_n * sb_n, F + F_RED, tid);
  if (tid < kN) {
    // w'_n rounded to binary16 once; the state operand factor undoes the rounding
    const __half wh = __float2half_rn(wmax > 0.0f ? sc_n * sb_n / wmax : 0.0f);
    reinterpret_cast<__half*>(F + F_WH)[tid] = wh;
    const float whf = __half2float(wh);
    F[F_HF + tid] = whf > 0.0f ? sc_n / whf : 0.0f;
  }
  const float A2 = __ldg(p.A + hd) * kLog2e;
  const float bias = p.dt_bias ? __ldg(p.dt_bias + hd) : 0.0f;
  const float Dh = p.D ? __ldg(p.D + hd) : 0.0f;

  // ---- initial state: thread (row = n, quarter) holds p in [16 q4, 16 q4 + 16)
  float hs[16];
  {
    float* stage = reinterpret_cast<float*>(smem + OFF_STATE);  // P x N fp32 = 32 KB
    if (p.h0 && seg == 0) {
      const float4* src = reinterpret_cast<const float4*>(p.h0 + u * kP * kN);
      for (int i = tid; i < kP * kN / 4; i += kThreads) reinterpret_cast<float4*>(stage)[i] = src[i];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 16; ++j) hs[j] = (p.h0 && seg == 0) ? stage[(16 * q4 + j) * kN + row] : 0.0f;
  }
  const float hfac = F[F_HF + row];  // state -> MMA2 operand
  const float sbr = F[F_SB + row];
  const uint32_t tmem = tmem_slot;
  const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
  // tensor memory columns: CB, Y_diag, Y_off, state increments, and M as the
  // binary16 A operand of MMA1 (row t in lane t, two steps per column)
  const uint32_t T_CB = 0, T_YD = 128, T_YO = 192, T_ACC = 256, T_M = 320;

  // Warp roles in the decay-matrix phase.  Warp (rb = warp & 3, q4) owns rows
  // [32 rb, 32 rb + 32) and columns [32 q4, 32 q4 + 32) of M: the ten warps
  // with q4 <= rb form M (named barrier 1); the six blocks above the
  // diagonal are zero, written once here, and their warps take other work
  // meanwhile: kIssueWarp issues the Y_off and state MMAs, kFactorWarp forms
  // the next tile's per-step factors and loads the dt values of the tile
  // after it.
  const bool m_warp = q4 <= (warp & 3);
  if (!m_warp) {
    F[F_RM + q4 * kQ + row] = 0.0f;
    const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    tc::tmem_st16(tmem + t_lane + T_M + 16 * q4, z);
    tc::tmem_wait_st();
  }
  // raw dt of the tile starting at t (binary16 bits; 0 beyond the end)
  uint16_t dtr[4] = {0, 0, 0, 0};
  auto load_dt = [&](int64_t t) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dtr[i] = t + 4 * lane + i < t_end ? p.dt[(bb * L + t + 4 * lane + i) * H + hd] : (uint16_t)0;
  };
  auto factors_from_raw = [&](int buf, int ql_) {
    float dtv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) dtv[i] = h2f(dtr[i]);
    tile_factors(F, buf, ql_, dtv, bias, p.softplus, A2, wmax, lane);
  };

  // ---- tile 0: raw rows, per-step factors, state maximum
  fetch_tile(p, smem, bb, hd, t_beg, (int)min((int64_t)kQ, t_end - t_beg), tid);
  if (warp == kFactorWarp) {
    load_dt(t_beg);
    factors_from_raw(0, (int)min((int64_t)kQ, t_end - t_beg));
    if (t_beg + kQ < t_end) load_dt(t_beg + kQ);
  }
  auto state_max = [&]() {
    float hm = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) hm = fmaxf(hm, fabsf(hs[j] * hfac));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) hm = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, o));
    if (lane == 0) F[F_RED + 2 + warp] = hm;
  };
  state_max();
  tc::cp_async_wait_all();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();

  // CB = C' B^T of tile j (M = t, N = s, K = n) into T_CB once its operand
  // blocks have landed: tile 0's by thread 0 here, tile j + 1's by kIssueWarp
  // once tile j's decay matrix is formed, so that it runs during tile j's
  // epilogue
  auto issue_cb = [&](int64_t j) {
    if (!ops_wait(j)) {
      flags |= SSMQ_DEV_TIMEOUT;
      abort_flag = 1;
      return;
    }
    tc::fence_after();
    const uint32_t cb = s_base + OFF_OPS + (uint32_t)(j & 1) * kOpTile;
    const uint32_t id = tc::idesc_f16(kQ, kQ, false, false);
#pragma unroll
    for (int k0 = 0; k0 < kN; k0 += 16)
      tc::mma_f16(tmem + T_CB, tc::kmaj_desc(cb, k0, kN), tc::kmaj_desc(cb + kOpBlock, k0, kN), id,
                  k0 > 0);
    tc::mma_commit(&bars[0]);
  };
  if (tid == 0) issue_cb(0);

  uint32_t phase = 0;
  int fb = 0;  // buffer of this tile's per-step factors
  float s_tot = 0.0f;  // log2 decay over the work item (thread 0)
  for (int64_t t0 = t_beg; t0 < t_end; t0 += kQ, phase ^= 1u, fb ^= 1) {
    const int ql = (int)min((int64_t)kQ, t_end - t0);
    const int64_t j = (t0 - t_beg) / kQ;  // tile of the work item
    const uint32_t cbuf = s_base + OFF_OPS + (uint32_t)(j & 1) * kOpTile;  // its C', then B
    const float* S2 = F + F_S2 + fb * kQ;
    const float* DW = F + F_DW + fb * kQ;
    const float* WX = F + F_WX + fb * kQ;
    const float* ES = F + F_ES + fb * kQ;
    const float* CW = F + F_CW + fb * kQ;
    const float* CD = F + F_CD + fb * kQ;
    const float s_last = F[F_RED + 1];
    const int ex = norm_exp(F[F_RED] * p.x_bound);  // x_bound >= max |x_exact|
    const float xsc = pow2i(-ex);
    float hmax_all = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) hmax_all = fmaxf(hmax_all, F[F_RED + 2 + w]);
    const int eh = norm_exp(hmax_all);

    // ---- stage x (exact) and w x (hi / lo): thread -> (row s, 16 p)
    {
      const int s = 32 * (warp >> 2) + lane, part = warp & 3;
      const bool ok = s < ql;
      const uint4 xq = ok ? *reinterpret_cast<const uint4*>(smem + OFF_RX + s * kP +
                                                            16 * (part ^ (s & 3)))
                          : make_uint4(0, 0, 0, 0);
      const float ws = WX[s] * xsc;
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {  // 8 p per group
        const uint32_t w0 = grp ? xq.z : xq.x, w1 = grp ? xq.w : xq.y;
        float xv[8];
        uint32_t ox[4], oh[4], ol[4];
        if (p.xfmt == SSMQ_X_INT8_GROUP) {
          const uint32_t x0 = w0 ^ 0x80808080u, x1 = w1 ^ 0x80808080u;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            xv[k] = s8_to_f32(x0, k);
            xv[4 + k] = s8_to_f32(x1, k);
          }
          ox[0] = h2_bits(s8x2_to_h2(x0, 0, 1));
          ox[1] = h2_bits(s8x2_to_h2(x0, 2, 3));
          ox[2] = h2_bits(s8x2_to_h2(x1, 0, 1));
          ox[3] = h2_bits(s8x2_to_h2(x1, 2, 3));
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            xv[k] = x_exact((w0 >> (8 * k)) & 0xFFu, p.xfmt, p.se_shift);
            xv[4 + k] = x_exact((w1 >> (8 * k)) & 0xFFu, p.xfmt, p.se_shift);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) ox[k] = pack_h2(xv[2 * k], xv[2 * k + 1]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) split_h2(ws * xv[2 * k], ws * xv[2 * k + 1], oh[k], ol[k]);
        const uint32_t off = tc::mnmaj_off(16 * part + 8 * grp, s, kP);
        *reinterpret_cast<uint4*>(smem + OFF_X + off) = make_uint4(ox[0], ox[1], ox[2], ox[3]);
        *reinterpret_cast<uint4*>(smem + OFF_XH + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
        *reinterpret_cast<uint4*>(smem + OFF_XL + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
      }
    }
    // ---- stage the state for Y_off: h'' = h sC_n / w'_n, normalised, binary16
    {
      const float f = hfac * pow2i(-eh);
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        uint32_t oh[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) oh[k] = pack_h2(hs[8 * grp + 2 * k] * f, hs[8 * grp + 2 * k + 1] * f);
        const uint32_t off = tc::mnmaj_off(16 * q4 + 8 * grp, row, kP);
        *reinterpret_cast<uint4*>(smem + OFF_HH + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
      }
    }
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();  // (B): operands staged, raw buffer consumed

    // ---- fetch the next tile's raw rows while this one runs
    const bool has_next = t0 + kQ < t_end;
    if (tid == 0) s_tot += s_last;
    if (has_next) fetch_tile(p, smem, bb, hd, t0 + kQ, (int)min((int64_t)kQ, t_end - t0 - kQ), tid);

    // ---- CB is in the tensor pipe already; kIssueWarp queues MMA2 (Y_off)
    // and MMA3 (state, hi + lo), which run while the M warps form M
    if (warp == kIssueWarp) {
      if (lane == 0) {
        tc::fence_after();
        if (!ops_wait(j)) {
          flags |= SSMQ_DEV_TIMEOUT;
          abort_flag = 1;
        } else {
          const uint32_t id_y = tc::idesc_f16(kQ, kP, false, true);
          const uint32_t id_s = tc::idesc_f16(kN, kP, true, true);
#pragma unroll
          for (int k0 = 0; k0 < kN; k0 += 16)
            tc::mma_f16(tmem + T_YO, tc::kmaj_desc(cbuf, k0, kN),
                        tc::mnmaj_desc(s_base + OFF_HH, k0, kP), id_y, k0 > 0);
#pragma unroll
          for (int k0 = 0; k0 < kQ; k0 += 16)
            tc::mma_f16(tmem + T_ACC, tc::mnmaj_desc(cbuf + kOpBlock, k0, kN),
                        tc::mnmaj_desc(s_base + OFF_XH, k0, kP), id_s, k0 > 0);
#pragma unroll
          for (int k0 = 0; k0 < kQ; k0 += 16)
            tc::mma_f16(tmem + T_ACC, tc::mnmaj_desc(cbuf + kOpBlock, k0, kN),
                        tc::mnmaj_desc(s_base + OFF_XL, k0, kP), id_s, 1u);
          tc::mma_commit(&bars[2]);
        }
      }
      __syncwarp();
    } else if (warp == kFactorWarp && has_next) {
      // the next tile's per-step factors (other buffer), then the dt values
      // of the tile after it
      factors_from_raw(fb ^ 1, (int)min((int64_t)kQ, t_end - t0 - kQ));
      if (t0 + 2 * kQ < t_end) load_dt(t0 + 2 * kQ);
    }

    if (m_warp) {
      if (!tc::mbar_wait(&bars[0], phase, kWaitLimit)) {
        flags |= SSMQ_DEV_TIMEOUT;
        abort_flag = 1;
      }
      tc::fence_after();
      // ---- M = CB * exp(S_t - S_s) * delta_s * w_max, row-normalised, s <= t
      // (thread: row t, columns s in [32 q4, 32 q4 + 32)).  Strictly below
      // the diagonal exp(S_t - S_s) = exp(S_t - S_p) exp(S_p - S_s) with p
      // the block's last step, both factors <= 1 (no overflow, underflow only
      // of negligible terms), and the row factor is applied with the
      // normalisation; on the diagonal block each element takes its own
      // exponential unless the block's S spread allows one more factoring.
      float mv[32];
      float rt = 1.0f;  // row factor still to apply to mv
      {
        const int t = row, s0 = 32 * q4, rb = warp & 3;
        float rmax = 0.0f;
        {
          float v[32];
          tc::tmem_ld32(tmem + t_lane + T_CB + s0, v);
          const float st = S2[t];
          if (q4 < rb) {
            rt = ex2_sfu(st - S2[s0 + 31]);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 c4 = *reinterpret_cast<const float4*>(CW + s0 + 4 * j4);
              const float cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float m = v[4 * j4 + e] * cw[e];
                mv[4 * j4 + e] = m;
                rmax = fmaxf(rmax, fabsf(m));
              }
            }
            rmax *= rt;
          } else if (F[F_BS + fb * 4 + q4] < 90.0f) {
            // diagonal block, S spread below 2^90: exp(S_t - S_s) =
            // exp(S_t - S_m) exp(S_m - S_s) with m the block's first step (both
            // factors within 2^+-90, the products far from fp32 overflow)
            const float sm = S2[s0];
            rt = ex2_sfu(st - sm);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 c4 = *reinterpret_cast<const float4*>(CD + s0 + 4 * j4);
              const float cd[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float m = s0 + 4 * j4 + e <= t ? v[4 * j4 + e] * cd[e] : 0.0f;
                mv[4 * j4 + e] = m;
                rmax = fmaxf(rmax, fabsf(m));
              }
            }
            rmax *= rt;
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int s = s0 + j;
              const float m = s <= t ? v[j] * ex2_sfu(st - S2[s]) * DW[s] * wmax : 0.0f;
              mv[j] = m;
              rmax = fmaxf(rmax, fabsf(m));
            }
          }
        }
        F[F_RM + q4 * kQ + t] = rmax;
      }
      tc::named_sync(1, 320);  // (C): row maxima published (the M warps)
      {
        const int t = row;
        const float rm = fmaxf(fmaxf(F[F_RM + t], F[F_RM + kQ + t]),
                               fmaxf(F[F_RM + 2 * kQ + t], F[F_RM + 3 * kQ + t]));
        const int et = norm_exp(rm);
        const float sc = pow2i(-et) * rt;
        if (q4 == 0) F[F_RS + t] = pow2i(et);
        uint32_t o[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = pack_h2(mv[2 * k] * sc, mv[2 * k + 1] * sc);
        tc::tmem_st16(tmem + t_lane + T_M + 16 * q4, o);
        tc::tmem_wait_st();
      }
      tc::fence_before();
      tc::named_sync(1, 320);  // (D): M in tensor memory
      // ---- MMA1 (Y_diag = M X)
      if (tid == 0 && !abort_flag) {
        tc::fence_after();
        const uint32_t id_y = tc::idesc_f16(kQ, kP, false, true);
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16)
          tc::mma_f16_ts(tmem + T_YD, tmem + T_M + k0 / 2, tc::mnmaj_desc(s_base + OFF_X, k0, kP),
                         id_y, k0 > 0);
        tc::mma_commit(&bars[1]);
      }
      __syncwarp();
      tc::named_arrive(3, kThreads);  // row scales published, CB read: T_CB free
    } else {
      tc::named_sync(3, kThreads);
      // tile j + 1's CB, queued behind this tile's MMAs (it runs during the
      // epilogue); kIssueWarp, not thread 0, waits for room in the MMA queue
      if (warp == kIssueWarp && lane == 0 && has_next && !abort_flag) issue_cb(j + 1);
      __syncwarp();
    }
    if (!tc::mbar_wait(&bars[1], phase, kWaitLimit) || !tc::mbar_wait(&bars[2], phase, kWaitLimit)) {
      flags |= SSMQ_DEV_TIMEOUT;
      abort_flag = 1;
    }
    tc::fence_after();
    // every MMA reading this tile's operand buffer is complete: tile j + 2's
    if (tid == 0 && j + 2 < n_tiles && !abort_flag) issue_ops(j + 2);

    // x scales of this thread's 16 columns
    float sxv[16];
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const float4 v = *reinterpret_cast<const float4*>(F + F_SX + 16 * q4 + 4 * j4);
      sxv[4 * j4] = v.x;
      sxv[4 * j4 + 1] = v.y;
      sxv[4 * j4 + 2] = v.z;
      sxv[4 * j4 + 3] = v.w;
    }
    // the three accumulators this thread reads (Y_diag, Y_off: row t; the
    // state increments: row n), one round trip to tensor memory
    float yd[16], yo[16], acc[16];
    tc::tmem_ld16x3(tmem + t_lane + T_YD + 16 * q4, tmem + t_lane + T_YO + 16 * q4,
                    tmem + t_lane + T_ACC + 16 * q4, yd, yo, acc);
    // ---- y = sx_p (Y_diag 2^e_t + D x_code) + exp(S_t) 2^e_h Y_off  (thread: row t, 16 p)
    {
      const int t = row;
      if (t < ql) {
        const float rs = F[F_RS + t], es = ES[t] * pow2i(eh);
        const int64_t yo_off = ((bb * L + t0 + t) * H + hd) * kP + 16 * q4;  // z
        // x of this row as exact binary16 values from the staged MMA operand
        uint32_t xw[8];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(smem + OFF_X +
                                                          tc::mnmaj_off(16 * q4 + 8 * i, t, kP));
          xw[4 * i] = v.x;
          xw[4 * i + 1] = v.y;
          xw[4 * i + 2] = v.z;
          xw[4 * i + 3] = v.w;
        }
        uint32_t zw[8];
        if (p.z) {
          const uint4* zr = reinterpret_cast<const uint4*>(p.z + yo_off);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint4 zz = __ldg(zr + i);
            zw[4 * i] = zz.x;
            zw[4 * i + 1] = zz.y;
            zw[4 * i + 2] = zz.z;
            zw[4 * i + 3] = zz.w;
          }
        }
        uint32_t out[8], qo[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const float2 xp = __half22float2(*reinterpret_cast<const __half2*>(&xw[j >> 1]));
          float2 zf = make_float2(0.0f, 0.0f);
          if (p.z) zf = __half22float2(*reinterpret_cast<const __half2*>(&zw[j >> 1]));
          float r2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int pj = j + e;
            float yv = fmaf(sxv[pj], fmaf(Dh, e ? xp.y : xp.x, yd[pj] * rs), es * yo[pj]);
            if (p.z) yv *= silu_f(e ? zf.y : zf.x);
            r2[e] = yv;
            if constexpr (kYQ) {
              // persistent-INT8 epilogue: the quantizer applied to the binary16 y,
              // by its reciprocal + magic-number route (exact division near a tie)
              const int pc = 16 * q4 + pj;
              const float v = h2f(f2h(yv)), ysc = F[F_YS + pc], yrs = F[F_YR + pc];
              const bool yok = F[F_YOK + pc] != 0.0f;
              const float yc = fminf(fmaxf(v * yrs, -127.0f), 127.0f);
              const float m = yc + 12582912.0f;
              const uint32_t c = (yok && yrs != 0.0f &&
                                  fabsf(yc - (m - 12582912.0f)) < 0.5f - 1.0f / 16384.0f &&
                                  fabsf(v) <= 3.402823466e38f)
                                     ? __float_as_uint(m) & 0xFFu
                                     : (uint32_t)quant_elem(v, ysc, yrs, yok, flags) & 0xFFu;
              qo[pj >> 2] |= c << (8 * (pj & 3));
            }
          }
          out[j / 2] = pack_half2(r2[0], r2[1]);
        }
        // y rows through shared memory (the state operands' buffers, free
        // once MMA3 is done): 16-byte chunks swizzled by row, no bank conflicts
        if (kYQ)
          *reinterpret_cast<uint4*>(smem + OFF_XL + t * kP + 16 * (q4 ^ ((t >> 1) & 3))) =
              make_uint4(qo[0], qo[1], qo[2], qo[3]);
        if (!kYQ || p.y) {
          uint8_t* yrow = smem + OFF_XH + t * (2 * kP);
          *reinterpret_cast<uint4*>(yrow + 16 * ((2 * q4) ^ (t & 7))) =
              make_uint4(out[0], out[1], out[2], out[3]);
          *reinterpret_cast<uint4*>(yrow + 16 * ((2 * q4 + 1) ^ (t & 7))) =
              make_uint4(out[4], out[5], out[6], out[7]);
        }
      }
      // the four warps of this row block write its 32 rows, whole 128-byte
      // (64-byte for int8) row segments per warp instruction
      const int rb = warp & 3, g = 32 * q4 + lane;
      tc::named_sync(4 + rb, 128);
      if (!kYQ || p.y) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int k = g + 128 * i, r = 32 * rb + k / 8, c = k % 8;
          if (r < ql) {
            const uint4 v = *reinterpret_cast<const uint4*>(smem + OFF_XH + r * (2 * kP) +
                                                             16 * (c ^ (r & 7)));
            *reinterpret_cast<uint4*>(p.y + ((bb * L + t0 + r) * H + hd) * kP + 8 * c) = v;
          }
        }
      }
      if (kYQ) {
        const int r = 32 * rb + g / 4, c = g % 4;
        if (r < ql) {
          const uint4 v = *reinterpret_cast<const uint4*>(smem + OFF_XL + r * kP +
                                                           16 * (c ^ ((r >> 1) & 3)));
          *reinterpret_cast<uint4*>(p.y_q + ((bb * L + t0 + r) * H + hd) * kP + 16 * c) = v;
        }
      }
    }
    // ---- state: h = exp(S_last) h + sB_n sx_p 2^e_x acc  (thread: row n, 16 p)
    {
      const float decay = ex2_sfu(s_last);
      const float f = sbr * pow2i(ex);
#pragma unroll
      for (int j = 0; j < 16; ++j) hs[j] = fmaf(decay, hs[j], f * sxv[j] * acc[j]);
    }
    // ---- next tile: state maximum, raw rows landed
    state_max();
    tc::cp_async_wait_all();
    tc::fence_before();
    if (__syncthreads_or(abort_flag)) break;  // (E): tile done
    tc::fence_after();
  }

  tc::cp_async_wait_all();  // no copy may land after the CTA has exited (abort path)
  // a copy issued but not waited for (the loop was left early) lands first
  if (tid == 0)
    for (int b = 0; b < 2; ++b)
      if (ops_n[b] && !tc::mbar_wait(&bars[3 + b], (ops_n[b] - 1u) & 1u, kWaitLimit))
        flags |= SSMQ_DEV_TIMEOUT;

  // ---- final state (P, N) through shared memory for coalesced stores: the
  // sequence's h_final, or a segment's local state for the second kernel
  float* fin = slot < 0 ? (p.h_final ? p.h_final + u * kP * kN : nullptr)
                        : p.seg_state + (int64_t)slot * kP * kN;
  if (slot >= 0 && tid == 0) p.seg_dec[slot] = s_tot;
  if (slot < 0 && tid == 0 && p.dec_final) p.dec_final[u] = s_tot;
  if (fin) {
    float* stage = reinterpret_cast<float*>(smem + OFF_STATE);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 16; ++j) stage[(16 * q4 + j) * kN + row] = hs[j];
    __syncthreads();
    float4* dst = reinterpret_cast<float4*>(fin);
    for (int i = tid; i < kP * kN / 4; i += kThreads) dst[i] = reinterpret_cast<float4*>(stage)[i];
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
  flag_status(p.status, flags);
}

// ---- segments of one sequence
// A sequence of the last SM round may be cut into kseg segments of seg_tiles
// tiles, each run by ssd_kernel from a zero state (segment 0 from h0).  The
// recurrence is linear in the state, so segment j's true state entering step
// t is its local one plus exp(S_t - S_j) h_start(j), S_j the cumulative decay
// at its first step, with h_start(j) = exp(dec_{j-1}) h_start(j-1) + loc_{j-1}
// from its predecessors' local final states loc and total decays dec
// (h_start(1) = loc_0, segment 0 having started from h0).  The
// missing output is the Y_off term of the segment's start state,
// exp(S_t - S_j) C_t h_start(j) (times silu(z_t) when gated): the second
// kernel adds it to y, rounding to binary16 once more, and forms h_final from
// the last segment.
constexpr int FX_C = 0;                       // C' blocks, K-major  [2]  64 KB
constexpr int FX_HH = FX_C + 2 * kOpBlock;    // start state operand      16 KB
constexpr int FX_ST = FX_HH + kN * kP * 2;    // start state fp32 (P, N)  32 KB
constexpr int FX_S2 = FX_ST + kP * kN * 4;    // S of the tile (log2)     [128]
constexpr int FX_HF = FX_S2 + kQ * 4;         // sC_n / w'_n              [128]
constexpr int FX_RED = FX_HF + kN * 4;        // reductions               [32]
constexpr int kFixSmem = FX_RED + 32 * 4;
constexpr uint32_t kFixCols = 64;

__global__ void __launch_bounds__(kThreads) ssd_fixup_kernel(const SsdParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(8) uint64_t bars[3];  // C' copies (two buffers), MMA
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // segments: CTA (seg - 1, sequence); carry-in mode (h_carry given): one CTA
  // per sequence, its whole length, from the given start state
  const bool carry = p.h_carry != nullptr;
  const int seg = carry ? 0 : 1 + (int)blockIdx.x;
  const int64_t slot0 = (int64_t)blockIdx.y * p.kseg;  // first segment slot of the unit
  const int64_t u = carry ? (int64_t)blockIdx.y : p.full + blockIdx.y;
  const int64_t H = p.H, L = p.L;
  const int64_t bb = u / H, hd = u % H;
  const int64_t g = hd * p.G / H;
  const int row = 32 * (warp & 3) + lane;
  const int q4 = warp >> 2;
  const uint32_t s_base = tc::smem_u32(smem);
  float* red = reinterpret_cast<float*>(smem + FX_RED);
  float* S2 = reinterpret_cast<float*>(smem + FX_S2);
  uint32_t flags = 0;

  if (warp == 0) tc::tmem_alloc(&tmem_slot, kFixCols);
  if (tid == 0) {
    tc::mbar_init(&bars[0], 1);
    tc::mbar_init(&bars[1], 1);
    tc::mbar_init(&bars[2], 1);
  }
  const uint8_t* ops_bg = p.ops + (bb * p.G + g) * p.ntiles * (int64_t)kOpTile;
  const int64_t tile_beg = carry ? 0 : (int64_t)seg * p.seg_tiles;
  const int64_t tile_end = carry ? p.ntiles : min(p.ntiles, tile_beg + p.seg_tiles);
  // C' of the segment's tile i -> buffer i & 1 (its (i >> 1)-th copy)
  auto issue_c = [&](int64_t i) {
    stream::expect_tx(&bars[i & 1], (uint32_t)kOpBlock);
    stream::bulk_g2s(smem + FX_C + (i & 1) * kOpBlock, ops_bg + (tile_beg + i) * kOpTile,
                     (uint32_t)kOpBlock, &bars[i & 1]);
  };
  uint32_t copies[2] = {0u, 0u};  // thread 0: copies issued per buffer
  __syncthreads();                // barriers initialised
  if (tid == 0) {
    issue_c(0);
    ++copies[0];
  }
  // state operand factor of the group (as in ssd_kernel)
  {
    float wmax, sc_n, sb_n;
    const __half wh = group_wprime(p, g, tid, red, wmax, sc_n, sb_n);
    if (tid < kN) {
      const float whf = __half2float(wh);
      reinterpret_cast<float*>(smem + FX_HF)[tid] = whf > 0.0f ? sc_n / whf : 0.0f;
    }
  }
  // h_start(seg) by the chain, elementwise; the last segment also forms h_final
  // and the sequence's total decay.  Carry-in mode: h_start is given.
  constexpr int kE = kP * kN / 4 / kThreads;  // float4 elements per thread
  float4* st = reinterpret_cast<float4*>(smem + FX_ST);
  if (carry) {
    const float4* hc = reinterpret_cast<const float4*>(p.h_carry + u * kP * kN);
#pragma unroll
    for (int i = 0; i < kE; ++i) st[tid + kThreads * i] = hc[tid + kThreads * i];
  } else {
    const float4* loc = reinterpret_cast<const float4*>(p.seg_state + slot0 * kP * kN);
    const float* dec = p.seg_dec + slot0;
    const bool last = seg == p.kseg - 1;
    constexpr int64_t kStride = kP * kN / 4;   // float4 per state
    auto fma4 = [](float d, float4 h, float4 l) {
      return make_float4(fmaf(d, h.x, l.x), fmaf(d, h.y, l.y), fmaf(d, h.z, l.z),
                         fmaf(d, h.w, l.w));
    };
    if (last && tid == 0 && p.dec_final) {
      float tot = 0.0f;
      for (int m = 0; m < p.kseg; ++m) tot += dec[m];
      p.dec_final[u] = tot;
    }
    // segment 0 ran from h0: its local state is already the true one
    float4 h[kE];
#pragma unroll
    for (int i = 0; i < kE; ++i) h[i] = loc[tid + kThreads * i];
#pragma unroll 2
    for (int m = 1; m < seg; ++m) {  // kE independent loads per step
      const float d = ex2_sfu(dec[m]);
#pragma unroll
      for (int i = 0; i < kE; ++i) h[i] = fma4(d, h[i], loc[m * kStride + tid + kThreads * i]);
    }
#pragma unroll
    for (int i = 0; i < kE; ++i) st[tid + kThreads * i] = h[i];
    if (last && p.h_final) {
      const float d = ex2_sfu(dec[seg]);
#pragma unroll
      for (int i = 0; i < kE; ++i)
        reinterpret_cast<float4*>(p.h_final + u * kP * kN)[tid + kThreads * i] =
            fma4(d, h[i], loc[seg * kStride + tid + kThreads * i]);
    }
  }
  __syncthreads();
  // operand h'' = h sC_n / w'_n 2^-e_h in binary16 (thread: row n, 16 p)
  int eh;
  {
    const float hfac = reinterpret_cast<const float*>(smem + FX_HF)[row];
    const float* st = reinterpret_cast<const float*>(smem + FX_ST);
    float hs[16];
    float hm = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      hs[j] = st[(16 * q4 + j) * kN + row] * hfac;
      hm = fmaxf(hm, fabsf(hs[j]));
    }
    eh = norm_exp(block_max(hm, red, tid));
    const float f = pow2i(-eh);
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
      uint32_t oh[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        oh[k] = pack_h2(hs[8 * grp + 2 * k] * f, hs[8 * grp + 2 * k + 1] * f);
      *reinterpret_cast<uint4*>(smem + FX_HH + tc::mnmaj_off(16 * q4 + 8 * grp, row, kP)) =
          make_uint4(oh[0], oh[1], oh[2], oh[3]);
    }
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();

  const uint32_t tmem = tmem_slot;
  const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
  const float A2 = __ldg(p.A + hd) * kLog2e;
  const float bias = p.dt_bias ? __ldg(p.dt_bias + hd) : 0.0f;
  const int64_t nt = tile_end - tile_beg;
  // raw dt of the segment's tile i (warp 0; binary16 bits, 0 beyond the end)
  uint16_t dtr[4] = {0, 0, 0, 0};
  auto load_dt = [&](int64_t i) {
    const int64_t tb = (tile_beg + i) * kQ;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      dtr[k] = tb + 4 * lane + k < L ? p.dt[(bb * L + tb + 4 * lane + k) * H + hd] : (uint16_t)0;
  };
  if (warp == 0) load_dt(0);
  // this thread's y (and z) row segment of the segment's tile i, loaded a
  // tile ahead (the rows are 10 KB apart: each load is its own transaction)
  const int t = row;
  uint4 yn[2], zn[2];
  auto load_yz = [&](int64_t i) {
    const int64_t tr = (tile_beg + i) * kQ + t;
    yn[0] = yn[1] = zn[0] = zn[1] = make_uint4(0u, 0u, 0u, 0u);
    if (tr < L) {
      const uint4* yr = reinterpret_cast<const uint4*>(p.y + ((bb * L + tr) * H + hd) * kP + 16 * q4);
      yn[0] = yr[0];
      yn[1] = yr[1];
      if (p.z) {
        const uint4* zr =
            reinterpret_cast<const uint4*>(p.z + ((bb * L + tr) * H + hd) * kP + 16 * q4);
        zn[0] = __ldg(zr);
        zn[1] = __ldg(zr + 1);
      }
    }
  };
  load_yz(0);
  float cum = 0.0f;  // S at the tile's start, from the segment's start
  bool failed = false;
  for (int64_t i = 0; i < nt; ++i) {
    const int64_t t0 = (tile_beg + i) * kQ;
    const int ql = (int)min((int64_t)kQ, L - t0);
    // the next tile's C' into the other buffer (the MMA that read it is done)
    if (tid == 0 && i + 1 < nt) {
      issue_c(i + 1);
      ++copies[(i + 1) & 1];
    }
    const int64_t off = ((bb * L + t0 + t) * H + hd) * kP + 16 * q4;
    const uint4 yv[2] = {yn[0], yn[1]}, zv[2] = {zn[0], zn[1]};
    if (i + 1 < nt) load_yz(i + 1);
    if (warp == 0) {
      float dtv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) dtv[k] = h2f(dtr[k]);
      float dl[4], sc[4], so, s_last;
      tile_decay(ql, dtv, bias, p.softplus, A2, lane, dl, sc, so, s_last);
      *reinterpret_cast<float4*>(S2 + 4 * lane) =
          make_float4(sc[0] + so, sc[1] + so, sc[2] + so, sc[3] + so);
      if (lane == 0) red[0] = s_last;
      if (i + 1 < nt) load_dt(i + 1);
    }
    if (tid == 0) {
      if (!tc::mbar_wait(&bars[i & 1], (uint32_t)(i >> 1) & 1u, kWaitLimit)) {
        flags |= SSMQ_DEV_TIMEOUT;
        failed = true;
      } else {
        tc::fence_after();
        const uint32_t cb = s_base + FX_C + (uint32_t)(i & 1) * kOpBlock;
        const uint32_t id_y = tc::idesc_f16(kQ, kP, false, true);
#pragma unroll
        for (int k0 = 0; k0 < kN; k0 += 16)
          tc::mma_f16(tmem, tc::kmaj_desc(cb, k0, kN), tc::mnmaj_desc(s_base + FX_HH, k0, kP), id_y,
                      k0 > 0);
        tc::mma_commit(&bars[2]);
      }
    }
    if (__syncthreads_or(failed)) break;  // S of the tile published, MMA issued
    if (!tc::mbar_wait(&bars[2], (uint32_t)i & 1u, kWaitLimit)) {
      flags |= SSMQ_DEV_TIMEOUT;
      failed = true;
    }
    if (__syncthreads_or(failed)) break;
    tc::fence_after();
    float v[16];
    tc::tmem_ld16(tmem + t_lane + 16 * q4, v);
    if (t < ql) {
      const float f = ex2_sfu(cum + S2[t]) * pow2i(eh);
      const uint32_t yw[8] = {yv[0].x, yv[0].y, yv[0].z, yv[0].w,
                              yv[1].x, yv[1].y, yv[1].z, yv[1].w};
      const uint32_t zw[8] = {zv[0].x, zv[0].y, zv[0].z, zv[0].w,
                              zv[1].x, zv[1].y, zv[1].z, zv[1].w};
      uint32_t out[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 yo = __half22float2(*reinterpret_cast<const __half2*>(&yw[k]));
        float c0 = f * v[2 * k], c1 = f * v[2 * k + 1];
        if (p.z) {
          const float2 zf = __half22float2(*reinterpret_cast<const __half2*>(&zw[k]));
          c0 *= silu_f(zf.x);
          c1 *= silu_f(zf.y);
        }
        out[k] = pack_h2(yo.x + c0, yo.y + c1);
      }
      uint4* yr = reinterpret_cast<uint4*>(p.y + off);
      yr[0] = make_uint4(out[0], out[1], out[2], out[3]);
      yr[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
    cum += red[0];
    tc::fence_before();
    __syncthreads();  // S and tensor memory free for the next tile
    tc::fence_after();
  }
  // carry-in mode: h_final += exp(S over the sequence) h_carry
  if (carry && p.h_final) {
    const float d = ex2_sfu(cum);
    float4* hf = reinterpret_cast<float4*>(p.h_final + u * kP * kN);
#pragma unroll
    for (int i = 0; i < kE; ++i) {
      const float4 c = st[tid + kThreads * i], h = hf[tid + kThreads * i];
      hf[tid + kThreads * i] = make_float4(fmaf(d, c.x, h.x), fmaf(d, c.y, h.y),
                                           fmaf(d, c.z, h.z), fmaf(d, c.w, h.w));
    }
  }
  // copies still in flight (the loop was left early) land before the CTA exits
  if (tid == 0)
    for (int b = 0; b < 2; ++b)
      if (copies[b] && !tc::mbar_wait(&bars[b], (copies[b] - 1u) & 1u, kWaitLimit))
        flags |= SSMQ_DEV_TIMEOUT;
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kFixCols);
  flag_status(p.status, flags);
}

#include "ssd_pipe.cuh"

}  // namespace

namespace {

constexpr int64_t kMaxSegSlots = 256;      // segment states a workspace holds at most
constexpr int64_t kDefaultMaxSegments = 32;  // segments per sequence when not given

int64_t seg_cap(const ssmq_ssd_args& a, int64_t ntiles) {
  if (a.max_segments == 1 || a.y_q || !a.y || ntiles < 2) return 1;
  return min(ntiles, a.max_segments > 0 ? (int64_t)a.max_segments : kDefaultMaxSegments);
}

// segment slots the workspace reserves: r k <= min(r cap, kMaxSegSlots), r <= units
int64_t seg_slots(const ssmq_ssd_args& a, int64_t ntiles) {
  const int64_t cap = seg_cap(a, ntiles);
  return cap < 2 ? 0 : min(kMaxSegSlots, a.batch * a.nheads * cap);
}

struct SegPlan {
  int64_t full;  // whole sequences (a multiple of the SM count)
  int64_t r;     // sequences cut into segments
  int kseg, seg_tiles;
};

// The last SM round of sequences (r = units mod SMs, or all units when fewer
// than the SMs) is cut into k segments each, r k <= SMs, so that round takes
// about 1/k of a sequence's time.
SegPlan seg_plan(const ssmq_ssd_args& a, int64_t ntiles, int sms) {
  const int64_t units = a.batch * a.nheads;
  const SegPlan none{units, 0, 1, (int)ntiles};
  const int64_t cap = seg_cap(a, ntiles);
  if (cap < 2 || sms <= 0) return none;
  const int64_t r = units >= sms ? units % sms : units;
  if (r == 0) return none;
  int64_t k = min(min((int64_t)sms / r, cap), kMaxSegSlots / r);
  if (k < 2) return none;
  const int64_t st = (ntiles + k - 1) / k;
  k = (ntiles + st - 1) / st;  // every segment holds at least one tile
  if (k < 2) return none;
  return SegPlan{units - r, r, (int)k, (int)st};
}

}  // namespace

size_t ssd_workspace_bytes(const ssmq_ssd_args& a) {
  if (a.seqlen <= 0 || a.batch <= 0 || a.nheads <= 0) return 0;
  const int64_t ntiles = (a.seqlen + kQ - 1) / kQ;
  const int64_t slots = seg_slots(a, ntiles);
  return (size_t)(a.batch * a.ngroups * ntiles) * (size_t)kOpTile +
         (size_t)slots * (size_t)(kP * kN * 4 + 4);
}

namespace {

// h_out[u][e] = fold over parts q of h <- exp2(dec[q][u]) h + h_end[q][u][e],
// from h = h_init[u][e] (0 when null); dec null means 0.
__global__ void state_chain_kernel(const float* __restrict__ h_end, const float* __restrict__ dec,
                                   int n_parts, int64_t units, int64_t elems,
                                   const float* h_init, float* h_out) {
  const int64_t n = units * elems;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t u = i / elems;
    float h = h_init ? h_init[i] : 0.0f;
    for (int q = 0; q < n_parts; ++q) {
      const float d = dec ? ex2_sfu(__ldg(dec + (int64_t)q * units + u)) : 1.0f;
      h = fmaf(d, h, __ldg(h_end + (int64_t)q * n + i));
    }
    h_out[i] = h;
  }
}

}  // namespace

cudaError_t launch_state_chain(const float* h_end, const float* dec, int n_parts, int64_t units,
                               int64_t elems, const float* h_init, float* h_out, cudaStream_t st) {
  const int64_t n = units * elems;
  if (n == 0) return cudaSuccess;
  const int64_t want = (n + 255) / 256, cap = (int64_t)sm_count() * 8;
  const int64_t blocks = want < cap ? want : cap;
  state_chain_kernel<<<(unsigned)blocks, 256, 0, st>>>(h_end, dec, n_parts, units, elems, h_init,
                                                       h_out);
  return cudaGetLastError();
}

namespace {

SsdParams make_params(const ssmq_ssd_args& a, void* ws) {
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
  p.y_q = a.y_q;
  p.y_group = a.y_group;
  p.y_scale = a.y_scale;
  p.n_y_groups = a.n_y_groups;
  p.h_final = a.h_final;
  p.dec_final = a.dec_final;
  p.status = a.status;
  p.ntiles = (a.seqlen + kQ - 1) / kQ;
  p.ops = static_cast<const uint8_t*>(ws);
  return p;
}

}  // namespace

cudaError_t launch_ssd(const ssmq_ssd_args& a, void* ws, cudaStream_t st) {
  const int64_t units = a.batch * a.nheads;
  if (units == 0) return cudaSuccess;
  if (a.seqlen == 0) {
    if (a.dec_final) {
      const cudaError_t e = cudaMemsetAsync(a.dec_final, 0, sizeof(float) * (size_t)units, st);
      if (e != cudaSuccess) return e;
    }
    if (!a.h_final) return cudaSuccess;
    const size_t bytes = sizeof(float) * (size_t)(units * a.headdim * a.dstate);
    return a.h0 ? cudaMemcpyAsync(a.h_final, a.h0, bytes, cudaMemcpyDeviceToDevice, st)
                : cudaMemsetAsync(a.h_final, 0, bytes, st);
  }
  SsdParams p = make_params(a, ws);
  const SegPlan sp = seg_plan(a, p.ntiles, sm_count());
  p.full = sp.full;
  p.kseg = sp.kseg;
  p.seg_tiles = sp.seg_tiles;
  const size_t ops_bytes = (size_t)(a.batch * a.ngroups * p.ntiles) * (size_t)kOpTile;
  p.seg_state = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ops_bytes);
  p.seg_dec = p.seg_state + seg_slots(a, p.ntiles) * kP * kN;
  ssd_operand_kernel<<<dim3((unsigned)p.ntiles, (unsigned)(a.batch * a.ngroups)), kThreads, 0, st>>>(
      p, static_cast<uint8_t*>(ws));
  // The single-schedule kernel by default; SSMQ_SSD_KERNEL=pipelined selects
  // the warp-role kernel for binary16 y (same bytes; slower on the 2.7B-shaped
  // workload so far: its roles run different code at once and each role has
  // one warp per scheduler, so instruction fetch and latency bound it)
  const char* kv = getenv("SSMQ_SSD_KERNEL");
  const bool classic = p.y_q || !(kv && strcmp(kv, "pipelined") == 0);
  const unsigned grid = (unsigned)(sp.full + sp.r * sp.kseg);
  cudaError_t e;
  if (classic) {
    auto kern = p.y_q ? ssd_kernel<true> : ssd_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, kSmemBytes, st>>>(p);
  } else {
    const bool se = p.xfmt == SSMQ_X_SOFTEDGE, gz = p.z != nullptr;
    auto kern = se ? (gz ? ssd_pipe_kernel<true, true> : ssd_pipe_kernel<true, false>)
                   : (gz ? ssd_pipe_kernel<false, true> : ssd_pipe_kernel<false, false>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pipe::kPSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, pipe::kPThreads, pipe::kPSmem, st>>>(p);
  }
  if (sp.r > 0) {
    e = cudaFuncSetAttribute(ssd_fixup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kFixSmem);
    if (e != cudaSuccess) return e;
    ssd_fixup_kernel<<<dim3((unsigned)(sp.kseg - 1), (unsigned)sp.r), kThreads, kFixSmem, st>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_ssd_carry_in(const ssmq_ssd_args& a, const float* h_carry, void* ws,
                                cudaStream_t st) {
  const int64_t units = a.batch * a.nheads;
  if (units == 0) return cudaSuccess;
  if (a.seqlen == 0) {  // h_final += h_carry
    if (!a.h_final) return cudaSuccess;
    return launch_state_chain(h_carry, nullptr, 1, units, a.headdim * a.dstate, a.h_final,
                              a.h_final, st);
  }
  SsdParams p = make_params(a, ws);
  p.h0 = nullptr;
  p.dec_final = nullptr;
  p.h_carry = h_carry;
  ssd_operand_kernel<<<dim3((unsigned)p.ntiles, (unsigned)(a.batch * a.ngroups)), kThreads, 0, st>>>(
      p, static_cast<uint8_t*>(ws));
  cudaError_t e = cudaFuncSetAttribute(ssd_fixup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kFixSmem);
  if (e != cudaSuccess) return e;
  ssd_fixup_kernel<<<dim3(1u, (unsigned)units), kThreads, kFixSmem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace ssmq
