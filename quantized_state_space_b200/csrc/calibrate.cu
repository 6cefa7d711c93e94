// Calibration on the device.
//
// Quamba2 (shd-paper.top card), method steps 1-2: per-channel activation
// statistics, then channels sorted by their magnitude and cut into clusters
// that share one scale.  Quamba-SE write-up 4.1: the soft-edge thresholds
// are the 5th and 99.9th percentiles of |x|, optionally blended into the
// running thresholds as alpha * new + (1 - alpha) * old.
//
//   cluster_rank_kernel   rank of every channel in (absmax, index) order by
//                         counting (n <= 65536), then its cluster and, for the
//                         last member of a cluster, the cluster's scale;
//   pct_hist / pct_select exact order statistics of |x| over the finite
//                         elements by radix selection on the magnitude bits:
//                         one 15-bit histogram pass for binary16 input (the
//                         bins are the values), three passes (15 + 8 + 8 bits)
//                         for fp32; the interpolation is done in double.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace ssmq {
namespace {

// ---- sort and cluster ----------------------------------------------------------

constexpr int kRankThreads = 256;
constexpr int kRankTile = 2048;

__global__ void __launch_bounds__(kRankThreads)
    cluster_rank_kernel(const float* __restrict__ absmax, int n, int k,
                        int32_t* __restrict__ cluster_of, float* __restrict__ scales,
                        uint32_t* status) {
  __shared__ uint64_t tile[kRankTile];
  const int i = blockIdx.x * kRankThreads + threadIdx.x;
  uint32_t flags = 0;
  // key: magnitude bits (the order of non-negative floats), then the index
  auto key_of = [&](int j) -> uint64_t {
    const float v = absmax[j];
    uint32_t b = __float_as_uint(v);
    if (!(v >= 0.0f) || !isfinite(v)) b = 0x7F800000u;  // flagged; sorts last
    return ((uint64_t)b << 32) | (uint32_t)j;
  };
  uint64_t ki = 0;
  if (i < n) {
    const float v = absmax[i];
    if (!(v >= 0.0f) || !isfinite(v)) flags |= SSMQ_DEV_NONFINITE;
    ki = key_of(i);
  }
  int rank = 0;
  for (int t0 = 0; t0 < n; t0 += kRankTile) {
    const int tn = min(kRankTile, n - t0);
    __syncthreads();
    for (int j = threadIdx.x; j < tn; j += kRankThreads) tile[j] = key_of(t0 + j);
    __syncthreads();
    if (i < n)
      for (int j = 0; j < tn; ++j) rank += tile[j] < ki;
  }
  if (i < n) {
    // cluster j holds sorted positions [floor(n j / k), floor(n (j + 1) / k))
    const int j = (int)((((int64_t)rank + 1) * k - 1) / n);
    cluster_of[i] = j;
    if (rank == (int)((int64_t)n * (j + 1) / k) - 1)
      scales[j] = __fdiv_rn(__uint_as_float((uint32_t)(ki >> 32)), 127.0f);
  }
  flag_status(status, flags);
}

// ---- percentiles of |x| ----------------------------------------------------------

constexpr int kMaxQ = 4;               // percentiles per call
constexpr int kTargets = 2 * kMaxQ;    // order statistics (k and k + 1 per percentile)
constexpr int kBins1 = 32768;          // 15-bit magnitude prefix
constexpr int kHistThreads = 1024;

struct PctCtrl {
  unsigned long long count;            // finite elements
  unsigned long long rank[kTargets];   // residual rank inside the current prefix
  uint32_t prefix[kTargets];           // magnitude bits selected so far
  double frac[kMaxQ];
  int nq;
  int pad;
};

struct PctWs {
  uint32_t h1[kBins1];
  uint32_t h2[kTargets][256];
  PctCtrl ctrl;
};

// magnitude bits of element i and whether it is finite
template <bool kF16>
__device__ __forceinline__ uint32_t mag_bits(const void* src, int64_t i, bool& fin) {
  if (kF16) {
    const uint32_t h = static_cast<const uint16_t*>(src)[i] & 0x7FFFu;
    fin = h < 0x7C00u;
    return h;
  }
  const uint32_t b = __float_as_uint(static_cast<const float*>(src)[i]) & 0x7FFFFFFFu;
  fin = b < 0x7F800000u;
  return b;
}

// Level 0: 15-bit prefix histogram of every finite element (binary16: the
// whole magnitude).  Level 1 / 2 (fp32): the next 8 bits of the elements whose
// prefix matches a target's.
template <bool kF16, int kLevel>
__global__ void __launch_bounds__(kHistThreads)
    pct_hist_kernel(const void* __restrict__ src, int64_t n, PctWs* ws) {
  extern __shared__ uint32_t sh[];
  const int nb = kLevel == 0 ? kBins1 : kTargets * 256;
  for (int b = threadIdx.x; b < nb; b += kHistThreads) sh[b] = 0u;
  uint32_t pre[kTargets];
  if (kLevel > 0)
#pragma unroll
    for (int t = 0; t < kTargets; ++t) pre[t] = ws->ctrl.prefix[t];
  const int nt = 2 * ws->ctrl.nq;
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * kHistThreads;
  int64_t i0 = 0;  // first element of the scalar loop below
  if (kLevel == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    // 16-byte loads (8 binary16 or 4 binary32 elements), then one shared
    // atomic per finite element; the scalar loop takes the remainder
    constexpr int kPer = kF16 ? 8 : 4;
    const int64_t nv = n / kPer;
    const uint4* v4 = static_cast<const uint4*>(src);
    for (int64_t v = (int64_t)blockIdx.x * kHistThreads + threadIdx.x; v < nv; v += stride) {
      const uint4 q = __ldg(v4 + v);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (kF16) {
          const uint32_t lo = w[k] & 0x7FFFu, hi = (w[k] >> 16) & 0x7FFFu;
          if (lo < 0x7C00u) atomicAdd(&sh[lo], 1u);
          if (hi < 0x7C00u) atomicAdd(&sh[hi], 1u);
        } else {
          const uint32_t m = w[k] & 0x7FFFFFFFu;
          if (m < 0x7F800000u) atomicAdd(&sh[m >> 16], 1u);
        }
      }
    }
    i0 = nv * kPer;
  }
  for (int64_t i = i0 + (int64_t)blockIdx.x * kHistThreads + threadIdx.x; i < n; i += stride) {
    bool fin;
    const uint32_t m = mag_bits<kF16>(src, i, fin);
    if (!fin) continue;
    if (kLevel == 0) {
      atomicAdd(&sh[kF16 ? m : m >> 16], 1u);
    } else {
      const uint32_t p = kLevel == 1 ? m >> 16 : m >> 8;
      const uint32_t dgt = kLevel == 1 ? (m >> 8) & 0xFFu : m & 0xFFu;
      for (int t = 0; t < nt; ++t)
        if (p == pre[t]) atomicAdd(&sh[t * 256 + dgt], 1u);
    }
  }
  __syncthreads();
  uint32_t* gh = kLevel == 0 ? ws->h1 : &ws->h2[0][0];
  for (int b = threadIdx.x; b < nb; b += kHistThreads)
    if (sh[b]) atomicAdd(gh + b, sh[b]);
}

// One CTA.  Level 0: count the finite elements, place the target ranks and
// find their 15-bit bins.  Level 1 / 2: extend each target's prefix by the
// next 8-bit digit.  At the last level the percentiles are formed:
// out[q] = fl32(v_k + frac (v_k+1 - v_k)), and, when thr is given, the
// soft-edge thresholds are updated from out[0] (low) and out[1] (high).
struct PctArgs {
  double q[kMaxQ];
};

template <bool kF16, int kLevel>
__global__ void __launch_bounds__(kHistThreads)
    pct_select_kernel(PctWs* ws, const PctArgs qa, int nq, float* out, float* thr,
                      float alpha) {
  __shared__ unsigned long long part[kHistThreads];
  PctCtrl& c = ws->ctrl;
  const int tid = threadIdx.x;
  constexpr bool kLast = kF16 ? kLevel == 0 : kLevel == 2;
  if (kLevel == 0) {
    // bins per thread: 32; inclusive prefix sums of the per-thread totals
    constexpr int per = kBins1 / kHistThreads;
    unsigned long long mine = 0;
    for (int b = 0; b < per; ++b) mine += ws->h1[tid * per + b];
    part[tid] = mine;
    __syncthreads();
    for (int o = 1; o < kHistThreads; o <<= 1) {
      const unsigned long long v = tid >= o ? part[tid - o] : 0ull;
      __syncthreads();
      part[tid] += v;
      __syncthreads();
    }
    const unsigned long long total = part[kHistThreads - 1];
    if (tid == 0) {
      c.count = total;
      c.nq = nq;
      for (int qi = 0; qi < nq; ++qi) {
        // position (m - 1) q / 100 in double; k clamped to [0, m - 1]
        const double pos = total ? (double)(total - 1) * (qa.q[qi] / 100.0) : 0.0;
        double kf = floor(pos);
        if (kf < 0.0) kf = 0.0;
        if (total && kf > (double)(total - 1)) kf = (double)(total - 1);
        const unsigned long long k = (unsigned long long)kf;
        c.frac[qi] = pos - kf;
        c.rank[2 * qi] = k;
        c.rank[2 * qi + 1] = (total && k + 1 < total) ? k + 1 : k;
      }
    }
    __syncthreads();
    unsigned long long rk[kTargets];
#pragma unroll
    for (int t = 0; t < kTargets; ++t) rk[t] = c.rank[t];
    __syncthreads();  // every thread has the ranks before any is rewritten
    // the thread whose bin range holds a target's rank finds the bin
    const unsigned long long lo = tid ? part[tid - 1] : 0ull, hi = part[tid];
    for (int t = 0; t < 2 * nq; ++t) {
      const unsigned long long r = rk[t];
      if (total && r >= lo && r < hi) {
        unsigned long long cum = lo;
        for (int b = 0; b < per; ++b) {
          const uint32_t h = ws->h1[tid * per + b];
          if (r < cum + h) {
            c.prefix[t] = (uint32_t)(tid * per + b);
            c.rank[t] = r - cum;
            break;
          }
          cum += h;
        }
      }
    }
  } else {
    // one warp per target: scan its 256 bins
    const int t = tid >> 5, lane = tid & 31;
    if (t < 2 * nq && c.count) {
      const uint32_t* h = ws->h2[t];
      unsigned long long cnt[8], sum = 0;
      for (int b = 0; b < 8; ++b) {
        cnt[b] = h[lane * 8 + b];
        sum += cnt[b];
      }
      unsigned long long incl = sum;
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned long long lo = incl - sum, r = c.rank[t];
      __syncwarp();
      if (r >= lo && r < incl) {
        unsigned long long cum = lo;
        for (int b = 0; b < 8; ++b) {
          if (r < cum + cnt[b]) {
            c.prefix[t] = (c.prefix[t] << 8) | (uint32_t)(lane * 8 + b);
            c.rank[t] = r - cum;
            break;
          }
          cum += cnt[b];
        }
      }
    }
  }
  if (!kLast) return;
  __syncthreads();
  if (tid == 0) {
    for (int qi = 0; qi < nq; ++qi) {
      double r = 0.0;
      if (c.count) {
        const uint32_t b0 = c.prefix[2 * qi], b1 = c.prefix[2 * qi + 1];
        const double vk = kF16 ? (double)__half2float(__ushort_as_half((uint16_t)b0))
                               : (double)__uint_as_float(b0);
        const double vk1 = kF16 ? (double)__half2float(__ushort_as_half((uint16_t)b1))
                                : (double)__uint_as_float(b1);
        r = vk + c.frac[qi] * (vk1 - vk);
      }
      out[qi] = (float)r;
    }
    if (thr) {
      // thresholds {scale, low, high}: blend, then scale = fl32(high / 63)
      const float lo = out[0], hi = out[1];
      const float L = alpha == 1.0f ? lo : (float)((double)alpha * lo + (1.0 - alpha) * thr[1]);
      const float H = alpha == 1.0f ? hi : (float)((double)alpha * hi + (1.0 - alpha) * thr[2]);
      thr[1] = L;
      thr[2] = H;
      thr[0] = (float)((double)H / 63.0);
    }
  }
}

template <bool kF16>
cudaError_t percentile_t(const void* src, int64_t n, const double* q, int nq, float* out,
                         float* thr, float alpha, void* workspace, cudaStream_t st) {
  PctWs* ws = static_cast<PctWs*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(PctWs), st);
  if (e != cudaSuccess) return e;
  PctArgs a{};
  for (int i = 0; i < nq; ++i) a.q[i] = q[i];
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + kHistThreads * 16 - 1) / (kHistThreads * 16);
  const int64_t g = want < (int64_t)sms ? want : (int64_t)sms;
  const unsigned grid = (unsigned)(g > 0 ? g : 1);
  const size_t sh0 = kBins1 * sizeof(uint32_t), sh1 = kTargets * 256 * sizeof(uint32_t);
  e = cudaFuncSetAttribute(pct_hist_kernel<kF16, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sh0);
  if (e != cudaSuccess) return e;
  pct_hist_kernel<kF16, 0><<<grid, kHistThreads, sh0, st>>>(src, n, ws);
  pct_select_kernel<kF16, 0><<<1, kHistThreads, 0, st>>>(ws, a, nq, out, thr, alpha);
  if (!kF16) {
    pct_hist_kernel<false, 1><<<grid, kHistThreads, sh1, st>>>(src, n, ws);
    pct_select_kernel<false, 1><<<1, kHistThreads, 0, st>>>(ws, a, nq, out, thr, alpha);
    // level 2 reuses the digit histograms
    e = cudaMemsetAsync(ws->h2, 0, sizeof(ws->h2), st);
    if (e != cudaSuccess) return e;
    pct_hist_kernel<false, 2><<<grid, kHistThreads, sh1, st>>>(src, n, ws);
    pct_select_kernel<false, 2><<<1, kHistThreads, 0, st>>>(ws, a, nq, out, thr, alpha);
  }
  return cudaGetLastError();
}

// Scratch of the allocation-free entry points: a static device array (module
// globals exist once per device context), sized exactly for one call.
constexpr size_t kPctWsBytes = (sizeof(PctWs) + 255) / 256 * 256 + 256;
__device__ __align__(256) uint8_t g_pct_scratch[kPctWsBytes];

}  // namespace

// Device address of each device's copy of the array, resolved by the first
// call made while that device is current (a host-side stand-in is all the
// symbol name gives host code).  Racing first calls store the same value.
static constexpr int kMaxDevices = 64;
static std::atomic<void*> g_scratch_addr[kMaxDevices];

void* percentile_static_scratch(size_t need, cudaError_t* err) {
  *err = cudaSuccess;
  if (need > kPctWsBytes) return nullptr;  // caller reports the size mismatch
  int dev = -1;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  void* p = cached ? g_scratch_addr[dev].load(std::memory_order_acquire) : nullptr;
  if (p) return p;
  *err = cudaGetSymbolAddress(&p, g_pct_scratch);  // the current device's copy
  if (*err != cudaSuccess) return nullptr;
  if (cached) g_scratch_addr[dev].store(p, std::memory_order_release);
  return p;
}

// workspace: the histograms and control block, then 256 bytes for the
// percentile values of the soft-edge update
size_t percentile_workspace_bytes() { return (sizeof(PctWs) + 255) / 256 * 256 + 256; }
float* percentile_scratch_out(void* ws) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + (sizeof(PctWs) + 255) / 256 * 256);
}
int percentile_max_q() { return kMaxQ; }

cudaError_t launch_percentile_abs(const void* src, bool f16, int64_t n, const double* q, int nq,
                                  float* out, float* thr, float alpha, void* workspace,
                                  cudaStream_t st) {
  return f16 ? percentile_t<true>(src, n, q, nq, out, thr, alpha, workspace, st)
             : percentile_t<false>(src, n, q, nq, out, thr, alpha, workspace, st);
}

cudaError_t launch_cluster_by_absmax(const float* absmax, int n, int k, int32_t* cluster_of,
                                     float* scales, uint32_t* status, cudaStream_t st) {
  cluster_rank_kernel<<<(n + kRankThreads - 1) / kRankThreads, kRankThreads, 0, st>>>(
      absmax, n, k, cluster_of, scales, status);
  return cudaGetLastError();
}

}  // namespace ssmq
