// Pipelined SSD kernel (binary16 y): included inside ssd.cu's anonymous
// namespace, after ssd_kernel, whose decomposition, operand layouts and
// arithmetic it keeps operation for operation (so its y and final state equal
// ssd_kernel's bit for bit).  What changes is the schedule.
//
// The recurrence couples 128-step tiles only through the fp32 state:
//   h_j = exp(S_last) h_{j-1} + ACC_j,   Y_off_j = C'_j h_{j-1}.
// Everything else of tile j (CB_j, the decay-weighted M_j, Y_diag_j = M_j X_j,
// the state increment ACC_j = B_j^T (w X)_j and the staging of x_j) does not
// depend on the state, so it can run a tile ahead.  The CTA is split into
// warp roles that work on different tiles at once and hand tiles to each
// other through mbarriers; the tensor core, driven by one thread, runs
// ACC_j, YD_j, YO_j and CB_{j+1} back to back while the CUDA cores form
// M_{j+1}, stage x_{j+1}, update the state and write y_j.
//
// Warp w reads TMEM lanes 32 (w % 4) .. (its lane quarter q = w % 4):
//   warps 0-7   M role: M_j from CB_j (TMEM) -> TMEM (A operand of YD_j);
//               thread = row t; the causal 32-column blocks 0 .. q of a row
//               are split between warps q and q + 4 (at most two each), two
//               passes (the row maximum, exchanged through shared memory,
//               then the normalised binary16 values)
//   warps 8-11  Y role: y_j from YD_j, YO_j (thread = row t), each thread
//               writing its row's 128 bytes
//   warps 12-19 S role: the state h (thread = row n and 32 of the 64 p in
//               registers), its maximum, the binary16 operand HH_{j+1}; and,
//               right after the state update (when ACC_j has freed the w x
//               buffers), the x operands of tile j + 1 (exact, double-
//               buffered, and w x as binary16 high / residual parts) from the
//               raw codes loaded before the wait
//   warp 20     per-step factors of each tile (delta, S, w, the decay
//               factors) and the operand-block copies
//   warp 21     lane 0 issues every MMA: CB_{j+1} as soon as M_j has read
//               CB_j, then ACC_j, YD_j, YO_j
// Every wait is bounded; a wait that gives up raises SSMQ_DEV_TIMEOUT and
// the shared abort word, which ends every role's loop; the CTA then waits
// (bounded) for its copies and MMAs in flight before it frees TMEM and exits.

namespace pipe {

constexpr int kPThreads = 704;
constexpr int W_Y = 8, W_S = 12, W_FAC = 20, W_MMA = 21;
// shared memory (bytes, dynamic)
constexpr int P_OPS = 0;                      // 2 x 64 KB operand blocks (C', B) of tiles
constexpr int P_X = P_OPS + 2 * kOpTile;      // x exact [s][p] MN-major, 2 x 16 KB (tile j in j & 1)
constexpr int P_XH = P_X + 2 * kQ * kP * 2;   // w x high                        16 KB
constexpr int P_XL = P_XH + kQ * kP * 2;      // w x residual                    16 KB
constexpr int P_HH = P_XL + kQ * kP * 2;      // state operand  [n][p] MN-major  16 KB
constexpr int P_F = P_HH + kN * kP * 2;       // fp32 scalars below
// the final state (P x N fp32, 32 KB) passes through P_XH .. P_XL at the end
// per-tile factor buffers (two, tile j in j & 1), floats
constexpr int FB_S2 = 0;          // S_t log2(e) within the tile    [128]
constexpr int FB_DW = 128;        // delta_s                        [128]
constexpr int FB_WX = 256;        // w_s = exp2(S_last - S_s) delta_s
constexpr int FB_ES = 384;        // exp2(S_t)
constexpr int FB_CW = 512;        // exp2(S_p(s) - S_s) delta_s w_max, p(s) = s | 31
constexpr int FB_CD = 640;        // exp2(S_m(s) - S_s) delta_s w_max, m(s) = s & ~31
constexpr int FB_BS = 768;        // S spread per 32-step block     [4]
constexpr int FB_WM = 772;        // max w_s of the tile
constexpr int FB_SL = 773;        // S_last
constexpr int FB_SIZE = 776;
constexpr int G_FB = 0;                       // 2 factor buffers
constexpr int G_RS = G_FB + 2 * FB_SIZE;      // row scale 2^e_t of M_j  [2][128]
constexpr int G_EH = G_RS + 2 * kQ;           // state normalisation exponent of HH_j [2] (int)
constexpr int G_HF = G_EH + 4;                // sC_n / w'_n              [128]
constexpr int G_SB = G_HF + kN;               // sB_n                     [128]
constexpr int G_SX = G_SB + kN;               // x scale per p            [64]
constexpr int G_RED = G_SX + kP;              // reductions               [32]
constexpr int G_RMX = G_RED + 32;             // M row maxima of the two warps of a quarter [2][128]
constexpr int G_END = G_RMX + 2 * kQ;
constexpr int kPSmem = P_F + G_END * 4;
static_assert(kPSmem + 1024 <= 232448, "shared memory of one CTA");
static_assert(P_XL + kQ * kP * 2 - P_XH >= kP * kN * 4, "final state staging");

// TMEM columns
constexpr uint32_t T_CB = 0, T_M = 128, T_YD = 192, T_YO = 256, T_ACC = 320;

// mbarriers (static shared memory), index
enum {
  B_OPS0 = 0, B_OPS1,   // operand block of a tile landed (bytes)
  B_CB,                 // CB_j complete (tcgen05.commit)
  B_ACC,                // ACC_j complete
  B_YD,                 // YD_j complete (and every earlier MMA)
  B_YO,                 // YO_j complete
  B_M,                  // M_j in TMEM (8 M warps)
  B_STAGE,              // X_j, XH_j, XL_j staged (8 S warps)
  B_HH,                 // HH_j staged (8 S warps)
  B_YFREE,              // Y role done reading YD_j, YO_j (4 Y warps)
  B_ACCFREE,            // S role done reading ACC_j (8 S warps)
  B_FAC0, B_FAC1,       // factors of a tile ready (factor warp)
  B_FFREE0, B_FFREE1,   // factor buffer free again (20 consumer warps)
  B_RS0, B_RS1,         // row scales of M_j written (8 M warps), buffer j & 1
  B_EH0, B_EH1,         // e_h of HH_j written (one S thread), buffer j & 1
  B_OPSF0, B_OPSF1,     // every MMA reading operand buffer j & 1 complete
  B_XF0, B_XF1,         // YD of the tile in x buffer j & 1 complete
  B_FINAL,              // every MMA complete (end)
  kNumBars
};
// A wait for phase k of an mbarrier is only correct while phase k + 1 has not
// completed (the parity would alias); every wait below is gated that way: the
// barrier's next phase needs something the waiting role does after the wait.
constexpr uint32_t kFacConsumers = 20;  // M 8 + Y 4 + S 8

// Probes at most `limit` times, giving up early when another role aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity,
                                         const volatile int* abort_flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (tc::mbar_try(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  return false;
}

__device__ __forceinline__ void bar_arrive(uint64_t* bar) { stream::arrive(bar); }

// AND of `pred` over the `n` threads of named barrier `id` (all of them take
// part, so a role's warps leave a loop together and never leave one another
// waiting at a named barrier)
__device__ __forceinline__ bool named_and(uint32_t id, uint32_t n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

}  // namespace pipe

// kSE: x as soft-edge codes (else int8 codes); kZ: gated output.  The
// specialisations keep each role's code small: the roles run different code
// at the same time, so every instruction of a hot loop competes for the
// instruction cache.
template <bool kSE, bool kZ>
__global__ void __launch_bounds__(pipe::kPThreads, 1) ssd_pipe_kernel(const SsdParams p) {
  using namespace pipe;
  constexpr int kXF = kSE ? SSMQ_X_SOFTEDGE : SSMQ_X_INT8_GROUP;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ int abort_flag;
  float* F = reinterpret_cast<float*>(smem + P_F);
  volatile int* abort_v = &abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // work item: a whole (batch, head) sequence, or segment seg of one
  int64_t u, t_beg = 0, t_end = p.L;
  int seg = 0, slot = -1;
  if ((int64_t)blockIdx.x < p.full) {
    u = blockIdx.x;
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
  const int nt = (int)((t_end - t_beg + kQ - 1) / kQ);
  const uint32_t s_base = tc::smem_u32(smem);
  uint32_t flags = 0;
  auto fail = [&]() {
    flags |= SSMQ_DEV_TIMEOUT;
    *abort_v = 1;
  };

  // ---- per-CTA constants (as ssd_kernel)
  float sc_n = 0.0f, sb_n = 0.0f;
  if (tid < kN) {
    const int si = (int)g * (kN / p.gs) + tid / p.gs;
    sc_n = __ldg(p.C_scale + si);
    sb_n = __ldg(p.B_scale + si);
    F[G_SB + tid] = sb_n;
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
    F[G_SX + tid] = sx;
  }
  if (tid == 0) abort_flag = 0;
  if (warp == 0) tc::tmem_alloc(&tmem_slot, 512);
  if (tid == 0) {
    tc::mbar_init(&bars[B_OPS0], 1);
    tc::mbar_init(&bars[B_OPS1], 1);
    tc::mbar_init(&bars[B_CB], 1);
    tc::mbar_init(&bars[B_ACC], 1);
    tc::mbar_init(&bars[B_YD], 1);
    tc::mbar_init(&bars[B_YO], 1);
    tc::mbar_init(&bars[B_M], 8);
    tc::mbar_init(&bars[B_STAGE], 8);
    tc::mbar_init(&bars[B_HH], 8);
    tc::mbar_init(&bars[B_YFREE], 4);
    tc::mbar_init(&bars[B_ACCFREE], 8);
    tc::mbar_init(&bars[B_FAC0], 1);
    tc::mbar_init(&bars[B_FAC1], 1);
    tc::mbar_init(&bars[B_FFREE0], kFacConsumers);
    tc::mbar_init(&bars[B_FFREE1], kFacConsumers);
    tc::mbar_init(&bars[B_RS0], 8);
    tc::mbar_init(&bars[B_RS1], 8);
    tc::mbar_init(&bars[B_EH0], 1);
    tc::mbar_init(&bars[B_EH1], 1);
    tc::mbar_init(&bars[B_OPSF0], 1);
    tc::mbar_init(&bars[B_OPSF1], 1);
    tc::mbar_init(&bars[B_XF0], 1);
    tc::mbar_init(&bars[B_XF1], 1);
    tc::mbar_init(&bars[B_FINAL], 1);
  }
  __syncthreads();
  const float wmax = block_max(sc_n * sb_n, F + G_RED, tid);
  if (tid < kN) {
    const __half wh = __float2half_rn(wmax > 0.0f ? sc_n * sb_n / wmax : 0.0f);
    const float whf = __half2float(wh);
    F[G_HF + tid] = whf > 0.0f ? sc_n / whf : 0.0f;
  }
  const float A2 = __ldg(p.A + hd) * kLog2e;
  const float bias = p.dt_bias ? __ldg(p.dt_bias + hd) : 0.0f;
  const float Dh = p.D ? __ldg(p.D + hd) : 0.0f;
  const uint8_t* ops_bg = p.ops + (bb * p.G + g) * p.ntiles * (int64_t)kOpTile;
  const int64_t tile0 = t_beg / kQ;
  const uint32_t tmem = tmem_slot;
  // operand block of tile j -> buffer j & 1 (the (j >> 1)-th copy into it)
  auto issue_ops = [&](int j) {
    stream::expect_tx(&bars[B_OPS0 + (j & 1)], (uint32_t)kOpTile);
    stream::bulk_g2s(smem + P_OPS + (j & 1) * kOpTile, ops_bg + (tile0 + j) * kOpTile,
                     (uint32_t)kOpTile, &bars[B_OPS0 + (j & 1)]);
  };
  int ops_issued = 0;  // warp 12 lane 0
  tc::fence_before();
  __syncthreads();  // constants and the TMEM address published
  tc::fence_after();

  if (warp < W_Y) {
    // =================================================================== M
    const int q = warp & 3, half = warp >> 2, t = 32 * q + lane;
    const uint32_t t_lane = (uint32_t)(32 * q) << 16;
    // this warp's blocks [cb0, cb1) of the causal blocks 0 .. q
    const int nb0 = (q + 2) >> 1;
    const int cb0 = half ? nb0 : 0, cb1 = half ? q + 1 : nb0;
    if (half == 0) {  // column blocks above the diagonal stay zero
      const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      for (int cb = q + 1; cb < 4; ++cb) tc::tmem_st16(tmem + t_lane + T_M + 16 * cb, z);
      tc::tmem_wait_st();
    }
    for (int j = 0; j < nt; ++j) {
      const int fb = j & 1;
      const float* FB = F + G_FB + fb * FB_SIZE;
      const bool ok = wait_bar(&bars[B_FAC0 + fb], (uint32_t)(j >> 1) & 1u, abort_v) &&
                      wait_bar(&bars[B_CB], (uint32_t)j & 1u, abort_v);
      if (!named_and(4, 256, ok)) {  // the M warps leave together
        fail();
        break;
      }
      tc::fence_after();
      const float st = FB[FB_S2 + t];
      const float* S2 = FB + FB_S2;
      const float* CW = FB + FB_CW;
      const float* CD = FB + FB_CD;
      const float* DW = FB + FB_DW;
      // block cb's row factor and mode (0 below the diagonal, 1 diagonal
      // factored, 2 diagonal per element), exactly as ssd_kernel's blocks
      auto block_mode = [&](int cb, float& rt) {
        rt = 1.0f;
        if (cb < q) {
          rt = ex2_sfu(st - S2[32 * cb + 31]);
          return 0;
        }
        if (FB[FB_BS + cb] < 90.0f) {
          rt = ex2_sfu(st - S2[32 * cb]);
          return 1;
        }
        return 2;
      };
      auto block_vals = [&](int cb, int mode, float (&mv)[32]) {
        tc::tmem_ld32(tmem + t_lane + T_CB + 32 * cb, mv);
        const int s0 = 32 * cb;
        if (mode != 2) {
          const float* fac = (mode == 0 ? CW : CD) + s0;
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 c4 = *reinterpret_cast<const float4*>(fac + 4 * j4);
            mv[4 * j4] *= c4.x;
            mv[4 * j4 + 1] *= c4.y;
            mv[4 * j4 + 2] *= c4.z;
            mv[4 * j4 + 3] *= c4.w;
          }
          if (mode == 1) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (s0 + jj > t) mv[jj] = 0.0f;
          }
        } else {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int s = s0 + jj;
            mv[jj] = s <= t ? mv[jj] * ex2_sfu(st - S2[s]) * DW[s] * wmax : 0.0f;
          }
        }
      };
      // pass 0: this warp's blocks' maximum, combined with the other warp of
      // the quarter through shared memory; pass 1: the normalised binary16
      // values (one loop body for both, to keep the code small)
      float rm = 0.0f;
      int et = 0;
      bool stop = false;  // uniform over the M warps (a named-barrier result)
      const int nbw = cb1 - cb0;
#pragma unroll 1
      for (int it = 0; it < 2 * nbw + 1; ++it) {
        if (it == nbw) {
          F[G_RMX + half * kQ + t] = rm;
          tc::named_sync(4, 256);
          rm = fmaxf(F[G_RMX + t], F[G_RMX + kQ + t]);
          et = norm_exp(rm);
          // M_{j-1} has been read by YD_{j-1} before M_j is written
          const bool ok2 = j == 0 || wait_bar(&bars[B_YD], (uint32_t)(j - 1) & 1u, abort_v);
          if (!named_and(4, 256, ok2)) {  // also: the maxima are read before they are rewritten
            fail();
            stop = true;
            break;
          }
          continue;
        }
        const int pass = it > nbw, cb = cb0 + (pass ? it - nbw - 1 : it);
        float rt, mv[32];
        const int mode = block_mode(cb, rt);
        block_vals(cb, mode, mv);
        if (!pass) {
          float mx = 0.0f;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) mx = fmaxf(mx, fabsf(mv[jj]));
          rm = fmaxf(rm, mode == 2 ? mx : mx * rt);
        } else {
          const float sc = pow2i(-et) * rt;
          uint32_t o[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = pack_h2(mv[2 * k] * sc, mv[2 * k + 1] * sc);
          tc::tmem_st16(tmem + t_lane + T_M + 16 * cb, o);
        }
      }
      if (stop) break;
      if (half == 0) F[G_RS + fb * kQ + t] = pow2i(et);
      tc::tmem_wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) {
        bar_arrive(&bars[B_M]);
        bar_arrive(&bars[B_RS0 + fb]);
        bar_arrive(&bars[B_FFREE0 + fb]);
      }
    }
  } else if (warp < W_S) {
    // =================================================================== Y
    const int q = warp - W_Y, t = 32 * q + lane;
    const uint32_t t_lane = (uint32_t)(32 * q) << 16;
    for (int j = 0; j < nt; ++j) {
      const int fb = j & 1;
      const float* FB = F + G_FB + fb * FB_SIZE;
      const int64_t t0 = t_beg + (int64_t)j * kQ;
      const int ql = (int)min((int64_t)kQ, t_end - t0);
      const int64_t row_off = ((bb * L + t0 + t) * H + hd) * kP;
      const uint8_t* xrow = static_cast<const uint8_t*>(p.x) + row_off;
      // this row's x codes (an L2 hit: the staging fetched them a tile ago)
      // and z, one 16-column quarter ahead of their use
      uint4 xq = make_uint4(0u, 0u, 0u, 0u), z0 = xq, z1 = xq;
      auto load_q = [&](int qq, uint4& xv, uint4& za, uint4& zb) {
        if (t < ql) {
          xv = __ldg(reinterpret_cast<const uint4*>(xrow + 16 * qq));
          if (kZ) {
            const uint4* zr = reinterpret_cast<const uint4*>(p.z + row_off + 16 * qq);
            za = __ldg(zr);
            zb = __ldg(zr + 1);
          }
        }
      };
      load_q(0, xq, z0, z1);
      bool ok = wait_bar(&bars[B_FAC0 + fb], (uint32_t)(j >> 1) & 1u, abort_v) &&
                wait_bar(&bars[B_RS0 + fb], (uint32_t)(j >> 1) & 1u, abort_v) &&
                wait_bar(&bars[B_EH0 + fb], (uint32_t)(j >> 1) & 1u, abort_v) &&
                wait_bar(&bars[B_YD], (uint32_t)j & 1u, abort_v) &&
                wait_bar(&bars[B_YO], (uint32_t)j & 1u, abort_v);
      if (!named_and(1, 128, ok)) {
        fail();
        break;
      }
      tc::fence_after();
      const float rs = F[G_RS + fb * kQ + t];
      const int eh = reinterpret_cast<const int*>(F + G_EH)[fb];
      const float es = FB[FB_ES + t] * pow2i(eh);
      uint16_t* ydst = p.y + row_off;
#pragma unroll 1
      for (int qq = 0; qq < 4; ++qq) {  // columns 16 qq .. 16 qq + 15
        uint4 xn = make_uint4(0u, 0u, 0u, 0u), zn0 = xn, zn1 = xn;
        if (qq < 3) load_q(qq + 1, xn, zn0, zn1);
        float yd[16], yo[16];
        tc::tmem_ld16(tmem + t_lane + T_YD + 16 * qq, yd);
        tc::tmem_ld16(tmem + t_lane + T_YO + 16 * qq, yo);
        const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
        const uint32_t zw[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
        const float* sxq = F + G_SX + 16 * qq;
        uint32_t out[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t w = xw[k >> 1];
          const float x0 = x_exact((w >> (16 * (k & 1))) & 0xFFu, kXF, p.se_shift);
          const float x1 = x_exact((w >> (16 * (k & 1) + 8)) & 0xFFu, kXF, p.se_shift);
          const float2 sx = *reinterpret_cast<const float2*>(sxq + 2 * k);
          float r2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float xv = e ? x1 : x0;
            float yv = fmaf(e ? sx.y : sx.x, fmaf(Dh, xv, yd[2 * k + e] * rs), es * yo[2 * k + e]);
            if (kZ) {
              const float2 zf = __half22float2(*reinterpret_cast<const __half2*>(&zw[k]));
              yv *= silu_f(e ? zf.y : zf.x);
            }
            r2[e] = yv;
          }
          out[k] = pack_half2(r2[0], r2[1]);
        }
        if (t < ql) {
          uint4* yq = reinterpret_cast<uint4*>(ydst + 16 * qq);
          yq[0] = make_uint4(out[0], out[1], out[2], out[3]);
          yq[1] = make_uint4(out[4], out[5], out[6], out[7]);
        }
        xq = xn;
        z0 = zn0;
        z1 = zn1;
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) {
        bar_arrive(&bars[B_YFREE]);
        bar_arrive(&bars[B_FFREE0 + fb]);
      }
    }
  } else if (warp < W_FAC) {
    // =================================================================== S
    const int sw = warp - W_S, q = sw & 3, half = sw >> 2, n = 32 * q + lane;
    const int p0 = 32 * half;  // this thread's columns p0 .. p0 + 31
    const uint32_t t_lane = (uint32_t)(32 * q) << 16;
    const float hfac = F[G_HF + n];
    const float sbr = F[G_SB + n];
    float hs[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
      hs[i] = (p.h0 && seg == 0) ? __ldg(p.h0 + u * kP * kN + (int64_t)(p0 + i) * kN + n) : 0.0f;
    // x operands of tile jj (exact into x buffer jj & 1, w x high / residual)
    // from raw codes xr[2] (items st_tid, st_tid + 256: row s, p in [16 part,
    // 16 part + 16)), with tile jj's per-step factors
    const int st_tid = 32 * sw + lane;
    auto load_x = [&](int jj, uint4 (&xr)[2]) {
      const int64_t tt = t_beg + (int64_t)jj * kQ;
      const int ql = (int)min((int64_t)kQ, t_end - tt);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int it = st_tid + 256 * i, s_ = it >> 2, part = it & 3;
        xr[i] = s_ < ql ? __ldg(reinterpret_cast<const uint4*>(
                              static_cast<const uint8_t*>(p.x) +
                              ((bb * L + tt + s_) * H + hd) * kP + 16 * part))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto stage_x = [&](int jj, const uint4 (&xr)[2]) {
      const float* FBs = F + G_FB + (jj & 1) * FB_SIZE;
      const int ex = norm_exp(FBs[FB_WM] * p.x_bound);
      const float xsc = pow2i(-ex);
      const uint32_t xb = P_X + (uint32_t)(jj & 1) * (kQ * kP * 2);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int it = st_tid + 256 * i, s_ = it >> 2, part = it & 3;
        const float ws = FBs[FB_WX + s_] * xsc;
#pragma unroll
        for (int grp = 0; grp < 2; ++grp) {
          const uint32_t w0 = grp ? xr[i].z : xr[i].x, w1 = grp ? xr[i].w : xr[i].y;
          float xv[8];
          uint32_t ox[4], oh[4], ol[4];
          if (!kSE) {
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
              xv[k] = x_exact((w0 >> (8 * k)) & 0xFFu, kXF, p.se_shift);
              xv[4 + k] = x_exact((w1 >> (8 * k)) & 0xFFu, kXF, p.se_shift);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) ox[k] = pack_h2(xv[2 * k], xv[2 * k + 1]);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) split_h2(ws * xv[2 * k], ws * xv[2 * k + 1], oh[k], ol[k]);
          const uint32_t off = tc::mnmaj_off(16 * part + 8 * grp, s_, kP);
          *reinterpret_cast<uint4*>(smem + xb + off) = make_uint4(ox[0], ox[1], ox[2], ox[3]);
          *reinterpret_cast<uint4*>(smem + P_XH + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
          *reinterpret_cast<uint4*>(smem + P_XL + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        }
      }
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) bar_arrive(&bars[B_STAGE]);
    };
    float s_tot = 0.0f;
    // exponent e_h of the state operand: the maximum of |h sC/w'| over the
    // whole state (the S warps), as ssd_kernel's state_max
    auto state_exp = [&]() {
      float hm = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) hm = fmaxf(hm, fabsf(hs[i] * hfac));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) hm = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, o));
      if (lane == 0) F[G_RED + 8 + sw] = hm;
      tc::named_sync(2, 256);
      float m = F[G_RED + 8];
#pragma unroll
      for (int i = 1; i < 8; ++i) m = fmaxf(m, F[G_RED + 8 + i]);
      tc::named_sync(2, 256);  // partials read before the next round writes them
      return norm_exp(m);
    };
    // HH = h sC_n / w'_n 2^-e_h, binary16, [n][p] MN-major
    auto stage_hh = [&](int eh) {
      const float f = hfac * pow2i(-eh);
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        uint32_t oh[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) oh[k] = pack_h2(hs[8 * grp + 2 * k] * f, hs[8 * grp + 2 * k + 1] * f);
        *reinterpret_cast<uint4*>(smem + P_HH + tc::mnmaj_off(p0 + 8 * grp, n, kP)) =
            make_uint4(oh[0], oh[1], oh[2], oh[3]);
      }
      tc::fence_async_smem();
      __syncwarp();
    };
    uint4 xr[2];
    load_x(0, xr);
    bool started = named_and(2, 256, wait_bar(&bars[B_FAC0], 0u, abort_v));
    if (started) {
      stage_x(0, xr);
      if (nt > 1) load_x(1, xr);
      const int eh = state_exp();
      if (n == 0 && half == 0) {
        reinterpret_cast<int*>(F + G_EH)[0] = eh;
        bar_arrive(&bars[B_EH0]);
      }
      stage_hh(eh);
      if (lane == 0) bar_arrive(&bars[B_HH]);
    } else {
      fail();
    }
    for (int j = 0; started && j < nt; ++j) {
      const int fb = j & 1;
      const float* FB = F + G_FB + fb * FB_SIZE;
      const bool ok = wait_bar(&bars[B_FAC0 + fb], (uint32_t)(j >> 1) & 1u, abort_v) &&
                      wait_bar(&bars[B_ACC], (uint32_t)j & 1u, abort_v);
      if (!named_and(2, 256, ok)) {
        fail();
        break;
      }
      tc::fence_after();
      const float s_last = FB[FB_SL];
      const int ex = norm_exp(FB[FB_WM] * p.x_bound);
      const float decay = ex2_sfu(s_last);
      const float f = sbr * pow2i(ex);
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        float acc[16];
        tc::tmem_ld16(tmem + t_lane + T_ACC + p0 + 16 * qq, acc);
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const float4 sx4 = *reinterpret_cast<const float4*>(F + G_SX + p0 + 16 * qq + 4 * i4);
          const float sx[4] = {sx4.x, sx4.y, sx4.z, sx4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 16 * qq + 4 * i4 + e;
            hs[i] = fmaf(decay, hs[i], f * sx[e] * acc[4 * i4 + e]);
          }
        }
      }
      if (n == 0 && half == 0) s_tot += s_last;
      tc::fence_before();
      __syncwarp();
      if (lane == 0) {
        bar_arrive(&bars[B_ACCFREE]);
        bar_arrive(&bars[B_FFREE0 + fb]);
      }
      if (j + 1 < nt) {
        // x operands of tile j + 1: its factors, and x buffer (j + 1) & 1 read
        // by YD_{j-1} (w x was read by ACC_j, complete)
        const bool ok1 = wait_bar(&bars[B_FAC0 + (fb ^ 1)], (uint32_t)((j + 1) >> 1) & 1u, abort_v) &&
                         (j < 1 || wait_bar(&bars[B_XF0 + (fb ^ 1)], (uint32_t)((j - 1) >> 1) & 1u,
                                            abort_v));
        if (!named_and(2, 256, ok1)) {
          fail();
          break;
        }
        stage_x(j + 1, xr);
        if (j + 2 < nt) load_x(j + 2, xr);
        const int eh = state_exp();
        const bool ok2 = wait_bar(&bars[B_YO], (uint32_t)j & 1u, abort_v);  // HH_j read by YO_j
        if (!named_and(2, 256, ok2)) {
          fail();
          break;
        }
        if (n == 0 && half == 0) {
          reinterpret_cast<int*>(F + G_EH)[(j + 1) & 1] = eh;
          bar_arrive(&bars[B_EH0 + ((j + 1) & 1)]);
        }
        stage_hh(eh);
        if (lane == 0) bar_arrive(&bars[B_HH]);
      }
    }
    // every MMA is complete (the MMA thread waited for all of them) before
    // the state staging area (XH, XL) is written
    if (!wait_bar(&bars[B_FINAL], 0u, abort_v)) fail();
    float* fin = slot < 0 ? (p.h_final ? p.h_final + u * kP * kN : nullptr)
                          : p.seg_state + (int64_t)slot * kP * kN;
    if (slot >= 0 && n == 0 && half == 0) p.seg_dec[slot] = s_tot;
    if (slot < 0 && n == 0 && half == 0 && p.dec_final) p.dec_final[u] = s_tot;
    if (fin) {
      float* stage = reinterpret_cast<float*>(smem + P_XH);
#pragma unroll
      for (int i = 0; i < 32; ++i) stage[(p0 + i) * kN + n] = hs[i];
      tc::named_sync(2, 256);
      float4* dst = reinterpret_cast<float4*>(fin);
      for (int i = 32 * sw + lane; i < kP * kN / 4; i += 256) dst[i] = reinterpret_cast<float4*>(stage)[i];
    }
  } else if (warp == W_FAC) {
    // =========================================================== factors
    uint16_t dtr[4] = {0, 0, 0, 0};
    auto load_dt = [&](int j) {
      const int64_t tt = t_beg + (int64_t)j * kQ;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dtr[i] = tt + 4 * lane + i < t_end ? p.dt[(bb * L + tt + 4 * lane + i) * H + hd] : (uint16_t)0;
    };
    if (lane == 0) {
      issue_ops(0);
      ++ops_issued;
      if (nt > 1) {
        issue_ops(1);
        ++ops_issued;
      }
    }
    load_dt(0);
    for (int j = 0; j < nt; ++j) {
      const int fb = j & 1;
      const bool ok = j < 2 || wait_bar(&bars[B_FFREE0 + fb], (uint32_t)((j - 2) >> 1) & 1u, abort_v);
      if (!__all_sync(0xffffffffu, ok)) {  // the warp leaves together (full-mask shuffles)
        fail();
        break;
      }
      const int ql = (int)min((int64_t)kQ, t_end - t_beg - (int64_t)j * kQ);
      float dtv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) dtv[i] = h2f(dtr[i]);
      float* FBw = F + G_FB + fb * FB_SIZE;
      // the same values as tile_factors (ssd_kernel), in this buffer layout
      {
        float dl[4], sc[4], off, s_last;
        tile_decay(ql, dtv, bias, p.softplus, A2, lane, dl, sc, off, s_last);
        float wmx = 0.0f;
        const float s_blk = __shfl_sync(0xffffffffu, sc[3] + off, lane | 7);
        const float s_beg = __shfl_sync(0xffffffffu, sc[0] + off, lane & ~7);
        float smax = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])) + off;
        float smin = fminf(fminf(sc[0], sc[1]), fminf(sc[2], sc[3])) + off;
#pragma unroll
        for (int o = 4; o >= 1; o >>= 1) {
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
          smin = fminf(smin, __shfl_xor_sync(0xffffffffu, smin, o));
        }
        if ((lane & 7) == 0) FBw[FB_BS + (lane >> 3)] = smax - smin;
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
        *reinterpret_cast<float4*>(FBw + FB_S2 + 4 * lane) = s2v;
        *reinterpret_cast<float4*>(FBw + FB_DW + 4 * lane) = dwv;
        *reinterpret_cast<float4*>(FBw + FB_WX + 4 * lane) = wxv;
        *reinterpret_cast<float4*>(FBw + FB_ES + 4 * lane) = esv;
        *reinterpret_cast<float4*>(FBw + FB_CW + 4 * lane) = cwv;
        *reinterpret_cast<float4*>(FBw + FB_CD + 4 * lane) = cdv;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) wmx = fmaxf(wmx, __shfl_xor_sync(0xffffffffu, wmx, o));
        if (lane == 0) {
          FBw[FB_WM] = wmx;
          FBw[FB_SL] = s_last;
        }
      }
      __syncwarp();
      if (lane == 0) bar_arrive(&bars[B_FAC0 + fb]);
      if (j + 1 < nt) load_dt(j + 1);
      // operand block of tile j + 1 into the buffer tile j - 1 used, once
      // YO_{j-1} (the last MMA reading it) is complete
      if (lane == 0 && j >= 1 && j + 1 < nt) {
        if (!wait_bar(&bars[B_OPSF0 + ((j - 1) & 1)], (uint32_t)((j - 1) >> 1) & 1u, abort_v)) {
          fail();
        } else {
          issue_ops(j + 1);
          ++ops_issued;
        }
      }
      if (__shfl_sync(0xffffffffu, *abort_v, 0)) break;
    }
    // copies issued land before the CTA may exit (the last two at most)
    if (lane == 0)
      for (int j = max(0, ops_issued - 2); j < ops_issued; ++j)
        if (!tc::mbar_wait(&bars[B_OPS0 + (j & 1)], (uint32_t)(j >> 1) & 1u, kWaitLimit))
          flags |= SSMQ_DEV_TIMEOUT;
  } else {
    // ================================================================ MMA
    if (lane == 0) {
      const uint32_t id_cb = tc::idesc_f16(kQ, kQ, false, false);
      const uint32_t id_y = tc::idesc_f16(kQ, kP, false, true);
      const uint32_t id_s = tc::idesc_f16(kN, kP, true, true);
      bool ok = wait_bar(&bars[B_OPS0], 0u, abort_v);
      if (ok) {
        tc::fence_after();
        const uint32_t cb = s_base + P_OPS;
#pragma unroll
        for (int k0 = 0; k0 < kN; k0 += 16)
          tc::mma_f16(tmem + T_CB, tc::kmaj_desc(cb, k0, kN), tc::kmaj_desc(cb + kOpBlock, k0, kN),
                      id_cb, k0 > 0);
        tc::mma_commit(&bars[B_CB]);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const uint32_t cbuf = s_base + P_OPS + (uint32_t)(j & 1) * kOpTile;
        // CB_{j+1}, as soon as M_j has read CB_j
        ok = wait_bar(&bars[B_M], (uint32_t)j & 1u, abort_v);
        if (!ok) break;
        if (j + 1 < nt) {
          ok = wait_bar(&bars[B_OPS0 + ((j + 1) & 1)], (uint32_t)((j + 1) >> 1) & 1u, abort_v);
          if (!ok) break;
          tc::fence_after();
          const uint32_t nb = s_base + P_OPS + (uint32_t)((j + 1) & 1) * kOpTile;
#pragma unroll
          for (int k0 = 0; k0 < kN; k0 += 16)
            tc::mma_f16(tmem + T_CB, tc::kmaj_desc(nb, k0, kN),
                        tc::kmaj_desc(nb + kOpBlock, k0, kN), id_cb, k0 > 0);
          tc::mma_commit(&bars[B_CB]);
        }
        // ACC_j = B_j^T (w X)_j, high and residual parts
        ok = wait_bar(&bars[B_STAGE], (uint32_t)j & 1u, abort_v) &&
             (j == 0 || wait_bar(&bars[B_ACCFREE], (uint32_t)(j - 1) & 1u, abort_v));
        if (!ok) break;
        tc::fence_after();
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16)
          tc::mma_f16(tmem + T_ACC, tc::mnmaj_desc(cbuf + kOpBlock, k0, kN),
                      tc::mnmaj_desc(s_base + P_XH, k0, kP), id_s, k0 > 0);
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16)
          tc::mma_f16(tmem + T_ACC, tc::mnmaj_desc(cbuf + kOpBlock, k0, kN),
                      tc::mnmaj_desc(s_base + P_XL, k0, kP), id_s, 1u);
        tc::mma_commit(&bars[B_ACC]);
        // YD_j = M_j X_j
        ok = j == 0 || wait_bar(&bars[B_YFREE], (uint32_t)(j - 1) & 1u, abort_v);
        if (!ok) break;
        tc::fence_after();
        const uint32_t xbuf = s_base + P_X + (uint32_t)(j & 1) * (kQ * kP * 2);
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16)
          tc::mma_f16_ts(tmem + T_YD, tmem + T_M + k0 / 2, tc::mnmaj_desc(xbuf, k0, kP), id_y,
                         k0 > 0);
        tc::mma_commit(&bars[B_YD]);
        tc::mma_commit(&bars[B_XF0 + (j & 1)]);  // x buffer j & 1 read completely
        // YO_j = C'_j HH_j
        ok = wait_bar(&bars[B_HH], (uint32_t)j & 1u, abort_v);
        if (!ok) break;
        tc::fence_after();
#pragma unroll
        for (int k0 = 0; k0 < kN; k0 += 16)
          tc::mma_f16(tmem + T_YO, tc::kmaj_desc(cbuf, k0, kN),
                      tc::mnmaj_desc(s_base + P_HH, k0, kP), id_y, k0 > 0);
        tc::mma_commit(&bars[B_YO]);
        tc::mma_commit(&bars[B_OPSF0 + (j & 1)]);  // operand buffer j & 1 read completely
      }
      if (!ok) fail();
      // every MMA issued is complete before TMEM is freed (and before the S
      // role reuses XH / XL for the final state)
      tc::mma_commit(&bars[B_FINAL]);
      if (!tc::mbar_wait(&bars[B_FINAL], 0u, kWaitLimit)) fail();
    }
    __syncwarp();
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
  flag_status(p.status, flags);
}
