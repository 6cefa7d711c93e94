// Symmetric int8 group quantizer and the three-mode soft-edge codec.
//
// Quamba-SE write-up (wmrh.cn) section 1: one scale factor maps floats onto
// the INT8 grid; sections 2.1-2.2: three modes (scale/4, scale, scale*4)
// chosen by comparing |v| with L and H, stored as 0xxxxxxx / 10xxxxxx /
// 11xxxxxx bytes.  Quamba2 abstract: one scale per cluster of x channels and
// per block of B/C states.
//
// The quantizer, the absmax pass and the encoder are HBM-bound streams: their
// input flows through the bulk-copy pipeline of stream.cuh (48 KB in flight
// per CTA, three CTAs per SM) and each consumer thread turns 16 elements into 16
// code bytes stored with one 16-byte store.  The decoder (1 byte in, 4 out)
// is store-bound and streams with plain 16-byte loads.
#include "common.cuh"
#include "internal.h"
#include "stream.cuh"
#include "fastdiv.h"
#include "quant_fast.cuh"

namespace ssmq {

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

namespace {

constexpr int kVec = 16;
constexpr int kThreads = 256;
constexpr int kMaxBlocks = 148 * 16;
enum { kPathRow = 0, kPathCol = 1, kPathGen = 2 };

template <bool kF16, typename Idx>
__device__ __forceinline__ void load16(const void* src, Idx e0, float (&v)[kVec]) {
  if (kF16) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + e0);
    const uint4 a = __ldg(p), b = __ldg(p + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + e0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = __ldg(p + i);
      v[4 * i] = f.x;
      v[4 * i + 1] = f.y;
      v[4 * i + 2] = f.z;
      v[4 * i + 3] = f.w;
    }
  }
}

template <bool kF16, typename Idx>
__device__ __forceinline__ float load1(const void* src, Idx e) {
  if (kF16) return h2f(static_cast<const uint16_t*>(src)[e]);
  return static_cast<const float*>(src)[e];
}

// Index geometry of a (outer, mid, inner) tensor: mid_of(e) = (e / inner) %
// mid is the group-map index of element e, col_of(e) = e % mid.  32-bit
// indices divide by multiply-shift (fastdiv.h), 64-bit ones by division.
template <typename Idx>
struct Geo;
template <>
struct Geo<uint32_t> {
  FastDiv inner, mid;
  __device__ __forceinline__ uint32_t mid_of(uint32_t e) const { return fmod_(fdiv(e, inner), mid); }
  __device__ __forceinline__ uint32_t col_of(uint32_t e) const { return fmod_(e, mid); }
};
template <>
struct Geo<uint64_t> {
  uint64_t inner, mid;
  __device__ __forceinline__ uint64_t mid_of(uint64_t e) const { return (e / inner) % mid; }
  __device__ __forceinline__ uint64_t col_of(uint64_t e) const { return e % mid; }
};
inline Geo<uint32_t> make_geo(uint32_t mid, uint32_t inner) {
  return Geo<uint32_t>{make_fastdiv(inner), make_fastdiv(mid)};
}
inline Geo<uint64_t> make_geo(uint64_t mid, uint64_t inner) { return Geo<uint64_t>{inner, mid}; }

// Per-CTA table of (scale, reciprocal) for small group counts, filled by
// the consumer threads in the pipeline's prologue (the producer's first
// copies are already in flight; the prologue ends with a consumer barrier).
constexpr int kMaxTab = 256;
__device__ __forceinline__ void fill_tab(const float* scales, int32_t n_groups, float2* tab) {
  for (int g = threadIdx.x; g < n_groups && g < kMaxTab; g += stream::kConsumers) {
    const float s = scales[g];
    const float r = __frcp_rn(s);
    tab[g] = make_float2(s, usable_recip(s, r) ? r : 0.0f);
  }
}
__device__ __forceinline__ float2 tab_get(const float2* tab, const float* scales, int g,
                                          int32_t n_groups) {
  return n_groups <= kMaxTab ? tab[g] : make_float2(__ldg(scales + g), 0.0f);
}


// One full 16-element vector of the static quantizer.
template <bool kF16, int kPath, typename Idx>
__device__ __forceinline__ void quant_vec(const float (&x)[kVec], Idx e0, const Geo<Idx>& geo,
                                          const int32_t* __restrict__ gmap, int32_t n_groups,
                                          const float* __restrict__ scales, const float2* tab,
                                          const int* ugrp, int8_t* __restrict__ q,
                                          uint32_t& flags) {
  int gu = -1, gv = -1;  // one group for each half of the vector, if known
  if (kPath == kPathRow) {
    gu = gv = __ldg(gmap + geo.mid_of(e0));
  } else if (kPath == kPathCol && ugrp) {
    const uint32_t u = (uint32_t)(geo.col_of(e0) >> 3);
    gu = ugrp[u];
    gv = ugrp[u + 1];
  }
  if ((unsigned)gu < (unsigned)n_groups && (unsigned)gv < (unsigned)n_groups) {
    const float2 sa = tab_get(tab, scales, gu, n_groups);
    const float2 sb = gv == gu ? sa : tab_get(tab, scales, gv, n_groups);
    uint4 o;
    if (sa.y != 0.0f && sb.y != 0.0f && quant16_fast(x, sa, sb, o)) {
      *reinterpret_cast<uint4*>(q + e0) = o;
      return;
    }
  }
  int r[kVec];
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int gh = i < kVec / 2 ? gu : gv;
    const int g = gh >= 0 || kPath == kPathRow
                      ? gh
                      : (kPath == kPathCol ? __ldg(gmap + geo.col_of(e0) + i)
                                           : __ldg(gmap + geo.mid_of(e0 + i)));
    const bool okg = (unsigned)g < (unsigned)n_groups;
    const float2 sr = okg ? tab_get(tab, scales, g, n_groups) : make_float2(0.0f, 0.0f);
    r[i] = quant_elem(x[i], sr.x, sr.y, okg, flags);
  }
  uint4 o;
  o.x = pack4(r[0], r[1], r[2], r[3]);
  o.y = pack4(r[4], r[5], r[6], r[7]);
  o.z = pack4(r[8], r[9], r[10], r[11]);
  o.w = pack4(r[12], r[13], r[14], r[15]);
  *reinterpret_cast<uint4*>(q + e0) = o;
}

// Dynamic shared memory: the pipeline's stages and barriers, then (absmax
// only) the per-CTA group accumulators.
template <bool kF16>
__host__ __device__ constexpr int acc_smem_offset() {
  return (stream::smem_bytes<kF16 ? 2 : 4>() + 15) / 16 * 16;
}

// Column path (inner == 1, mid % 16 == 0): groups of 8 consecutive columns
// that share one group id are marked in a per-CTA table (-1 otherwise); a
// vector's two halves look up their own entry.  ugrp_of says whether the
// table is used; fill_ugrp fills it in the prologue, like fill_tab.
constexpr int kMaxU = 2048;
__device__ __forceinline__ const int* ugrp_of(uint64_t mid, int* ug) {
  return mid / (kVec / 2) > (uint64_t)kMaxU ? nullptr : ug;
}
__device__ __forceinline__ void fill_ugrp(const int32_t* gmap, uint64_t mid, int* ug) {
  constexpr int kW = kVec / 2;
  const uint64_t nu = mid / kW;
  if (nu > (uint64_t)kMaxU) return;
  for (uint64_t u = threadIdx.x; u < nu; u += stream::kConsumers) {
    const int g0 = __ldg(gmap + u * kW);
    bool same = true;
    for (int i = 1; i < kW; ++i) same &= __ldg(gmap + u * kW + i) == g0;
    ug[u] = same ? g0 : -1;
  }
}

template <bool kF16, int kPath, typename Idx>
__global__ void __launch_bounds__(stream::kThreads)
    quant_static_kernel(const void* __restrict__ src, Idx n, Idx mid, const Geo<Idx> geo,
                        const int32_t* __restrict__ gmap, int32_t n_groups,
                        const float* __restrict__ scales, int8_t* __restrict__ q,
                        uint32_t* status, uint32_t wait_limit) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float2 tab[kMaxTab];
  __shared__ int ug_s[kPath == kPathCol ? kMaxU : 1];
  const int* ugrp = kPath == kPathCol ? ugrp_of((uint64_t)mid, ug_s) : nullptr;
  uint32_t flags = 0;
  auto vec = [&](const float(&x)[kVec], Idx e0) {
    quant_vec<kF16, kPath, Idx>(x, e0, geo, gmap, n_groups, scales, tab, ugrp, q, flags);
  };
  auto one = [&](float v, Idx e) {
    const int g = __ldg(gmap + geo.mid_of(e));
    const bool okg = (unsigned)g < (unsigned)n_groups;
    q[e] = (int8_t)quant_elem(v, okg ? __ldg(scales + g) : 0.0f, 0.0f, okg, flags);
  };
  auto pro = [&]() {
    fill_tab(scales, n_groups, tab);
    if (kPath == kPathCol) fill_ugrp(gmap, (uint64_t)mid, ug_s);
  };
  stream::run_part<kF16, Idx, decltype(vec)&, decltype(one)&, decltype(pro)&>(
      src, n, smem, (Idx)blockIdx.x, (Idx)gridDim.x, vec, one, flags, wait_limit, pro);
  flag_status(status, flags);
}

// Several static quantizations in one launch (same dtype, path and index
// width): job k owns CTAs [cta_beg, cta_end) of the grid and runs the
// pipeline over its tensor as CTA (blockIdx.x - cta_beg) of that range.
constexpr int kMaxJobs = kMaxQuantJobs;
template <typename Idx>
struct QJob {
  const void* src;
  Idx n, mid;
  Geo<Idx> geo;
  const int32_t* gmap;
  int32_t n_groups;
  const float* scales;
  int8_t* q;
  int cta_beg, cta_end;
};
template <typename Idx>
struct QJobs {
  QJob<Idx> j[kMaxJobs];
  int n;
};

template <bool kF16, int kPath, typename Idx>
__global__ void __launch_bounds__(stream::kThreads)
    quant_batch_kernel(const __grid_constant__ QJobs<Idx> jobs, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float2 tab[kMaxTab];
  __shared__ int ug_s[kPath == kPathCol ? kMaxU : 1];
  int k = 0;
  while (k + 1 < jobs.n && (int)blockIdx.x >= jobs.j[k].cta_end) ++k;
  const QJob<Idx>& J = jobs.j[k];
  const int* ugrp = kPath == kPathCol ? ugrp_of((uint64_t)J.mid, ug_s) : nullptr;
  uint32_t flags = 0;
  auto vec = [&](const float(&x)[kVec], Idx e0) {
    quant_vec<kF16, kPath, Idx>(x, e0, J.geo, J.gmap, J.n_groups, J.scales, tab, ugrp, J.q,
                                flags);
  };
  auto one = [&](float v, Idx e) {
    const int g = __ldg(J.gmap + J.geo.mid_of(e));
    const bool okg = (unsigned)g < (unsigned)J.n_groups;
    J.q[e] = (int8_t)quant_elem(v, okg ? __ldg(J.scales + g) : 0.0f, 0.0f, okg, flags);
  };
  auto pro = [&]() {
    fill_tab(J.scales, J.n_groups, tab);
    if (kPath == kPathCol) fill_ugrp(J.gmap, (uint64_t)J.mid, ug_s);
  };
  stream::run_part<kF16, Idx, decltype(vec)&, decltype(one)&, decltype(pro)&>(
      J.src, J.n, smem, (Idx)((int)blockIdx.x - J.cta_beg), (Idx)(J.cta_end - J.cta_beg), vec,
      one, flags, stream::kWaitLimit, pro);
  flag_status(status, flags);
}

// Per-group max |v| into `acc` (the scales buffer viewed as uint32 bit
// patterns: for non-negative floats the unsigned order is the float order).
template <bool kF16, int kPath, typename Idx>
__global__ void __launch_bounds__(stream::kThreads)
    absmax_kernel(const void* __restrict__ src, Idx n, const Geo<Idx> geo,
                  const int32_t* __restrict__ gmap, int32_t n_groups, unsigned* acc,
                  uint32_t* status, int use_smem) {
  extern __shared__ __align__(128) uint8_t smem[];
  unsigned* s_acc = reinterpret_cast<unsigned*>(smem + acc_smem_offset<kF16>());
  if (use_smem)
    for (int i = threadIdx.x; i < n_groups; i += blockDim.x) s_acc[i] = 0u;
  // (stream::run begins with a block barrier)
  unsigned* tgt = use_smem ? s_acc : acc;
  uint32_t flags = 0;
  int cur_g = -1;
  unsigned cur_m = 0u;
  auto push = [&](int g, float v) {
    if ((unsigned)g >= (unsigned)n_groups) {
      flags |= SSMQ_DEV_BAD_GROUP;
      return;
    }
    if (!isfinite(v)) {
      flags |= SSMQ_DEV_NONFINITE;
      return;
    }
    const unsigned a = __float_as_uint(fabsf(v));
    if (g != cur_g) {
      if (cur_g >= 0 && cur_m) atomicMax(tgt + cur_g, cur_m);
      cur_g = g;
      cur_m = a;
    } else {
      cur_m = max(cur_m, a);
    }
  };
  auto one = [&](float v, Idx e) { push(__ldg(gmap + geo.mid_of(e)), v); };
  if constexpr (kPath == kPathRow && kF16) {
    // a vector's 16 elements share one group: the largest magnitude pattern
    // of the vector by packed 16-bit maxima (for non-negative binary16 the
    // pattern order is the value order); a vector holding a non-finite
    // element (exponent bits all ones, found per pair as in the encoder)
    // takes the per-element definition
    auto vec = [&](const uint32_t(&w)[8], Idx e0) {
      const int g = __ldg(gmap + geo.mid_of(e0));
      uint32_t m = 0u, nf = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        nf |= (w[i] & 0x7C007C00u) + 0x04000400u;
        m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
      }
      if (nf & 0x80008000u) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          push(g, h2f((uint16_t)(w[i] & 0xFFFFu)));
          push(g, h2f((uint16_t)(w[i] >> 16)));
        }
        return;
      }
      push(g, h2f((uint16_t)max(m & 0xFFFFu, m >> 16)));
    };
    stream::run_part<true, Idx, decltype(vec)&, decltype(one)&, stream::NoPrologue, true>(
        src, n, smem, (Idx)blockIdx.x, (Idx)gridDim.x, vec, one, flags);
  } else {
  stream::run<kF16, Idx>(
      src, n, smem,
      [&](const float(&x)[kVec], Idx e0) {
        if (kPath == kPathRow) {
          // binary32: the largest magnitude bit pattern of the vector, or the
          // per-element definition when an element is not finite
          const int g = __ldg(gmap + geo.mid_of(e0));
          uint32_t m = 0u;
          bool nfv = false;
#pragma unroll
          for (int i = 0; i < kVec; ++i) {
            const uint32_t a = __float_as_uint(x[i]) & 0x7FFFFFFFu;
            nfv |= a >= 0x7F800000u;
            m = max(m, a);
          }
          if (nfv) {
#pragma unroll
            for (int i = 0; i < kVec; ++i) push(g, x[i]);
          } else {
            push(g, __uint_as_float(m));
          }
        } else if (kPath == kPathCol) {
          const Idx m0 = geo.col_of(e0);
#pragma unroll
          for (int i = 0; i < kVec; ++i) push(__ldg(gmap + m0 + i), x[i]);
        } else {
#pragma unroll
          for (int i = 0; i < kVec; ++i) push(__ldg(gmap + geo.mid_of(e0 + i)), x[i]);
        }
      },
      one, flags);
  }
  if (cur_g >= 0 && cur_m) atomicMax(tgt + cur_g, cur_m);
  if (use_smem) {
    __syncthreads();
    for (int i = threadIdx.x; i < n_groups; i += blockDim.x)
      if (s_acc[i]) atomicMax(acc + i, s_acc[i]);
  }
  flag_status(status, flags);
}

// scale_g = fl32(absmax_g / 127), in place over the accumulator.
__global__ void absmax_finalize_kernel(float* scales, int32_t n_groups) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g < n_groups) {
    const unsigned bits = reinterpret_cast<unsigned*>(scales)[g];
    scales[g] = __fdiv_rn(__uint_as_float(bits), 127.0f);
  }
}

template <typename Idx>
unsigned grid_for(Idx n) {
  const uint64_t nvec = ((uint64_t)n + kVec - 1) / kVec;
  uint64_t b = (nvec + kThreads - 1) / kThreads;
  if (b > (uint64_t)kMaxBlocks) b = kMaxBlocks;
  return (unsigned)(b ? b : 1);
}

// Launches a pipeline kernel with `smem` bytes of dynamic shared memory.
template <class... P, class... A>
cudaError_t launch_stream(void (*kern)(P...), uint64_t n, size_t smem, cudaStream_t st,
                          A... args) {
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<stream::grid_for(n, sm_count()), stream::kThreads, smem, st>>>(args...);
  return cudaGetLastError();
}

template <bool kF16, int kPath, typename Idx>
cudaError_t quantize_t(const void* src, Idx n, Idx mid, Idx inner, const int32_t* gmap,
                       int32_t n_groups, bool absmax, float* scales, int8_t* q,
                       uint32_t* status, cudaStream_t st) {
  constexpr size_t pipe = (size_t)acc_smem_offset<kF16>();
  const Geo<Idx> geo = make_geo(mid, inner);
  cudaError_t e = cudaSuccess;
  if (absmax) {
    e = cudaMemsetAsync(scales, 0, sizeof(float) * (size_t)n_groups, st);
    if (e != cudaSuccess) return e;
    const int use_smem = n_groups <= 8192;
    if (n > 0) {
      e = launch_stream(absmax_kernel<kF16, kPath, Idx>, (uint64_t)n,
                        pipe + (use_smem ? n_groups * sizeof(unsigned) : 0), st, src, n, geo,
                        gmap, n_groups, reinterpret_cast<unsigned*>(scales), status, use_smem);
      if (e != cudaSuccess) return e;
    }
    absmax_finalize_kernel<<<(n_groups + 255) / 256, 256, 0, st>>>(scales, n_groups);
  }
  if (n > 0)
    e = launch_stream(quant_static_kernel<kF16, kPath, Idx>, (uint64_t)n, pipe, st, src, n, mid,
                      geo, gmap, n_groups, (const float*)scales, q, status, stream::wait_limit());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// exact max |v| of every group (finite elements), no scale division
template <bool kF16, int kPath, typename Idx>
cudaError_t group_absmax_t(const void* src, Idx n, Idx mid, Idx inner, const int32_t* gmap,
                           int32_t n_groups, float* absmax, uint32_t* status, cudaStream_t st) {
  constexpr size_t pipe = (size_t)acc_smem_offset<kF16>();
  const Geo<Idx> geo = make_geo(mid, inner);
  cudaError_t e = cudaMemsetAsync(absmax, 0, sizeof(float) * (size_t)n_groups, st);
  if (e != cudaSuccess || n == 0) return e;
  const int use_smem = n_groups <= 8192;
  return launch_stream(absmax_kernel<kF16, kPath, Idx>, (uint64_t)n,
                       pipe + (use_smem ? n_groups * sizeof(unsigned) : 0), st, src, n, geo, gmap,
                       n_groups, reinterpret_cast<unsigned*>(absmax), status, use_smem);
}

template <bool kF16, typename Idx>
cudaError_t group_absmax_p(const void* src, Idx n, Idx mid, Idx inner, const int32_t* gmap,
                           int32_t n_groups, float* absmax, uint32_t* status, cudaStream_t st) {
  if (inner % kVec == 0)
    return group_absmax_t<kF16, kPathRow, Idx>(src, n, mid, inner, gmap, n_groups, absmax, status, st);
  if (inner == 1 && mid % kVec == 0)
    return group_absmax_t<kF16, kPathCol, Idx>(src, n, mid, inner, gmap, n_groups, absmax, status, st);
  return group_absmax_t<kF16, kPathGen, Idx>(src, n, mid, inner, gmap, n_groups, absmax, status, st);
}

template <bool kF16, typename Idx>
cudaError_t quantize_p(const void* src, Idx n, Idx mid, Idx inner, const int32_t* gmap,
                       int32_t n_groups, bool absmax, float* scales, int8_t* q,
                       uint32_t* status, cudaStream_t st) {
  if (inner % kVec == 0)
    return quantize_t<kF16, kPathRow, Idx>(src, n, mid, inner, gmap, n_groups, absmax, scales, q,
                                           status, st);
  if (inner == 1 && mid % kVec == 0)
    return quantize_t<kF16, kPathCol, Idx>(src, n, mid, inner, gmap, n_groups, absmax, scales, q,
                                           status, st);
  return quantize_t<kF16, kPathGen, Idx>(src, n, mid, inner, gmap, n_groups, absmax, scales, q,
                                         status, st);
}

// ---- soft-edge ---------------------------------------------------------------

template <bool kF16, typename Idx>
__global__ void __launch_bounds__(stream::kThreads)
    se_encode_kernel(const void* __restrict__ src, Idx n, float lo, float hi, SeSteps st,
                     uint8_t* __restrict__ codes, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t flags = 0;
  const bool fast_ok = st.rs[0] != 0.0f && st.rs[1] != 0.0f && st.rs[2] != 0.0f;
  stream::run<kF16, Idx>(
      src, n, smem,
      [&](const float(&x)[kVec], Idx e0) {
        uint4 fast;
        if (fast_ok && se16_fast(x, lo, hi, st, fast)) {
          *reinterpret_cast<uint4*>(codes + e0) = fast;
          return;
        }
        uint32_t wd[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          wd[k] = se_encode1(x[4 * k], lo, hi, st, flags) |
                  (se_encode1(x[4 * k + 1], lo, hi, st, flags) << 8) |
                  (se_encode1(x[4 * k + 2], lo, hi, st, flags) << 16) |
                  (se_encode1(x[4 * k + 3], lo, hi, st, flags) << 24);
        *reinterpret_cast<uint4*>(codes + e0) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      },
      [&](float v, Idx e) { codes[e] = (uint8_t)se_encode1(v, lo, hi, st, flags); }, flags);
  flag_status(status, flags);
}

// binary16 input: the code of every one of the 65536 bit patterns is
// computed once per CTA, exactly as se_encode1 defines it, into a 64 KB
// shared-memory table (by the consumers, while the producer's first copies
// are in flight); each element is then one table load.  A non-finite element
// (exponent bits all ones) is found per 32-bit pair: (w & 0x7C007C00) +
// 0x04000400 sets bit 15 of a half exactly when that half's exponent field
// is 0x1F.  Two CTAs per SM (64 KB table + 48 KB of stages each).
constexpr int kLutBytes = 65536;

// Four soft-edge codes with their payloads negated, byte by byte: a standard
// code (bit 7 clear) holds q mod 128 and becomes (128 - b) mod 128; a small
// or large code keeps its two mode bits and its 6-bit payload p becomes
// (64 - p) mod 64.  The per-byte differences never borrow across bytes.
__device__ __forceinline__ uint32_t neg_codes4(uint32_t w) {
  const uint32_t std = (0x80808080u - (w & 0x7F7F7F7Fu)) & 0x7F7F7F7Fu;
  const uint32_t spec = ((0x40404040u - (w & 0x3F3F3F3Fu)) & 0x3F3F3F3Fu) | (w & 0xC0C0C0C0u);
  const uint32_t sm = ((w & 0x80808080u) >> 7) * 0xFFu;  // 0xFF in each small / large byte
  return (std & ~sm) | (spec & sm);
}
constexpr int kLutCtasPerSm = 2;

template <typename Idx>
__global__ void __launch_bounds__(stream::kThreads, kLutCtasPerSm)
    se_encode_lut_kernel(const uint16_t* __restrict__ src, Idx n, float lo, float hi, SeSteps st,
                         uint8_t* __restrict__ codes, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* lut = smem;
  uint32_t flags = 0;
  // the table: the codes of the non-negative patterns 16 at a time by the
  // packed route (se16_fast); a run holding a non-finite pattern, or any run
  // when the steps do not allow the packed route, by se_encode1 element by
  // element (its flags discarded: a pattern in the table need not occur in
  // the data).  The negative patterns take the negated payloads
  // (neg_codes4): the mode depends on |v| only and the rounding and the
  // clamp are odd functions, so code(-v) carries -q in the same mode.
  const bool fast_ok = st.rs[0] != 0.0f && st.rs[1] != 0.0f && st.rs[2] != 0.0f;
  auto build = [&]() {
    uint32_t dummy = 0;
    for (int i = threadIdx.x; i < kLutBytes / 2 / kQVec; i += stream::kConsumers) {
      float x[kQVec];
#pragma unroll
      for (int k = 0; k < kQVec; ++k) x[k] = h2f((uint16_t)(kQVec * i + k));
      uint4 o;
      if (!(fast_ok && se16_fast(x, lo, hi, st, o))) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          w[k] = se_encode1(x[4 * k], lo, hi, st, dummy) |
                 (se_encode1(x[4 * k + 1], lo, hi, st, dummy) << 8) |
                 (se_encode1(x[4 * k + 2], lo, hi, st, dummy) << 16) |
                 (se_encode1(x[4 * k + 3], lo, hi, st, dummy) << 24);
        o = make_uint4(w[0], w[1], w[2], w[3]);
      }
      reinterpret_cast<uint4*>(lut)[i] = o;
      reinterpret_cast<uint4*>(lut + kLutBytes / 2)[i] =
          make_uint4(neg_codes4(o.x), neg_codes4(o.y), neg_codes4(o.z), neg_codes4(o.w));
    }
  };
  uint32_t nf = 0;  // bit 15 / 31 set by a non-finite half
  auto vec = [&](const uint32_t(&w)[8], Idx e0) {
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t a = w[2 * k], b = w[2 * k + 1];
      nf |= ((a & 0x7C007C00u) + 0x04000400u) | ((b & 0x7C007C00u) + 0x04000400u);
      const uint32_t c0 = lut[a & 0xFFFFu], c1 = lut[a >> 16];
      const uint32_t c2 = lut[b & 0xFFFFu], c3 = lut[b >> 16];
      o[k] = __byte_perm(__byte_perm(c0, c1, 0x0040), __byte_perm(c2, c3, 0x0040), 0x5410);
    }
    *reinterpret_cast<uint4*>(codes + e0) = make_uint4(o[0], o[1], o[2], o[3]);
  };
  auto one = [&](float v, Idx e) { codes[e] = (uint8_t)se_encode1(v, lo, hi, st, flags); };
  stream::run_part<true, Idx, decltype(vec)&, decltype(one)&, decltype(build)&, true>(
      src, n, smem + kLutBytes, (Idx)blockIdx.x, (Idx)gridDim.x, vec, one, flags,
      stream::kWaitLimit, build);
  if (nf & 0x80008000u) flags |= SSMQ_DEV_NONFINITE;
  flag_status(status, flags);
}

template <typename Idx>
__global__ void __launch_bounds__(kThreads)
    se_decode_kernel(const uint8_t* __restrict__ codes, Idx n, SeSteps st, float* __restrict__ out) {
  const Idx nvec = (n + kVec - 1) / kVec;
  for (Idx v = (Idx)blockIdx.x * kThreads + threadIdx.x; v < nvec; v += (Idx)gridDim.x * kThreads) {
    const Idx e0 = v * kVec;
    if (e0 + kVec <= n) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(codes + e0));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      float4* o = reinterpret_cast<float4*>(out + e0);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        o[k] = make_float4(se_decode(w[k] & 0xFFu, st), se_decode((w[k] >> 8) & 0xFFu, st),
                           se_decode((w[k] >> 16) & 0xFFu, st), se_decode(w[k] >> 24, st));
    } else {
      for (Idx e = e0; e < n; ++e) out[e] = se_decode(codes[e], st);
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const void* src, bool f16, int64_t outer, int64_t mid, int64_t inner,
                            const int32_t* gmap, int32_t n_groups, bool absmax, float* scales,
                            int8_t* q, uint32_t* status, cudaStream_t st) {
  const uint64_t n = (uint64_t)outer * (uint64_t)mid * (uint64_t)inner;
  if (n + 64 < (1ull << 32)) {
    const uint32_t n32 = (uint32_t)n, m32 = (uint32_t)mid, i32 = (uint32_t)inner;
    return f16 ? quantize_p<true, uint32_t>(src, n32, m32, i32, gmap, n_groups, absmax, scales, q,
                                            status, st)
               : quantize_p<false, uint32_t>(src, n32, m32, i32, gmap, n_groups, absmax, scales, q,
                                             status, st);
  }
  return f16 ? quantize_p<true, uint64_t>(src, n, (uint64_t)mid, (uint64_t)inner, gmap, n_groups,
                                          absmax, scales, q, status, st)
             : quantize_p<false, uint64_t>(src, n, (uint64_t)mid, (uint64_t)inner, gmap, n_groups,
                                           absmax, scales, q, status, st);
}

namespace {

int path_of(int64_t mid, int64_t inner) {
  return inner % kVec == 0 ? kPathRow : (inner == 1 && mid % kVec == 0 ? kPathCol : kPathGen);
}

// one launch for jobs idx[0..m) (same dtype, path and index width); CTAs in
// proportion to each job's tiles, one at least
template <bool kF16, int kPath, typename Idx>
cudaError_t batch_t(const QuantJob* jobs, const int* idx, int m, uint32_t* status,
                    cudaStream_t st) {
  QJobs<Idx> J{};
  J.n = m;
  uint64_t tiles[kMaxJobs], total = 0;
  for (int i = 0; i < m; ++i) {
    const QuantJob& q = jobs[idx[i]];
    const uint64_t n = (uint64_t)q.outer * (uint64_t)q.mid * (uint64_t)q.inner;
    tiles[i] = n / stream::kTileElems;
    total += tiles[i];
  }
  // one resident round of CTAs: floor shares (one at least), the rest to the
  // jobs with the most tiles per CTA; never more CTAs than tiles (but one)
  const uint64_t budget = (uint64_t)sm_count() * stream::kCtasPerSm;
  uint64_t cta[kMaxJobs], used = 0;
  for (int i = 0; i < m; ++i) {
    cta[i] = total ? budget * tiles[i] / total : 1;
    if (cta[i] < 1) cta[i] = 1;
    if (tiles[i] > 0 && cta[i] > tiles[i]) cta[i] = tiles[i];
    used += cta[i];
  }
  while (used < budget) {
    int best = -1;
    for (int i = 0; i < m; ++i)
      if (cta[i] < tiles[i] &&
          (best < 0 || tiles[i] * cta[best] > tiles[best] * cta[i]))
        best = i;
    if (best < 0) break;
    ++cta[best];
    ++used;
  }
  int beg = 0;
  for (int i = 0; i < m; ++i) {
    const QuantJob& q = jobs[idx[i]];
    const uint64_t n = (uint64_t)q.outer * (uint64_t)q.mid * (uint64_t)q.inner;
    const uint64_t c = cta[i];
    QJob<Idx>& d = J.j[i];
    d.src = q.src;
    d.n = (Idx)n;
    d.mid = (Idx)q.mid;
    d.geo = make_geo((Idx)q.mid, (Idx)q.inner);
    d.gmap = q.gmap;
    d.n_groups = q.n_groups;
    d.scales = q.scales;
    d.q = q.q;
    d.cta_beg = beg;
    beg += (int)c;
    d.cta_end = beg;
  }
  auto kern = quant_batch_kernel<kF16, kPath, Idx>;
  constexpr size_t smem = (size_t)acc_smem_offset<kF16>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)beg, stream::kThreads, smem, st>>>(J, status);
  return cudaGetLastError();
}

template <bool kF16, typename Idx>
cudaError_t batch_p(int path, const QuantJob* jobs, const int* idx, int m, uint32_t* status,
                    cudaStream_t st) {
  if (path == kPathRow) return batch_t<kF16, kPathRow, Idx>(jobs, idx, m, status, st);
  if (path == kPathCol) return batch_t<kF16, kPathCol, Idx>(jobs, idx, m, status, st);
  return batch_t<kF16, kPathGen, Idx>(jobs, idx, m, status, st);
}

}  // namespace

cudaError_t launch_quantize_batch(const QuantJob* jobs, int n_jobs, uint32_t* status,
                                  cudaStream_t st) {
  // group the non-empty jobs by (dtype, path, index width): one launch each
  bool done[kMaxJobs] = {};
  for (int a = 0; a < n_jobs; ++a) {
    const uint64_t na = (uint64_t)jobs[a].outer * (uint64_t)jobs[a].mid * (uint64_t)jobs[a].inner;
    if (done[a] || na == 0) continue;
    const int pa = path_of(jobs[a].mid, jobs[a].inner);
    const bool wa = na + 64 >= (1ull << 32);
    int idx[kMaxJobs], m = 0;
    for (int b = a; b < n_jobs; ++b) {
      const uint64_t nb =
          (uint64_t)jobs[b].outer * (uint64_t)jobs[b].mid * (uint64_t)jobs[b].inner;
      if (done[b] || nb == 0 || jobs[b].f16 != jobs[a].f16 ||
          path_of(jobs[b].mid, jobs[b].inner) != pa || (nb + 64 >= (1ull << 32)) != wa)
        continue;
      idx[m++] = b;
      done[b] = true;
    }
    const cudaError_t e =
        wa ? (jobs[a].f16 ? batch_p<true, uint64_t>(pa, jobs, idx, m, status, st)
                          : batch_p<false, uint64_t>(pa, jobs, idx, m, status, st))
           : (jobs[a].f16 ? batch_p<true, uint32_t>(pa, jobs, idx, m, status, st)
                          : batch_p<false, uint32_t>(pa, jobs, idx, m, status, st));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_group_absmax(const void* src, bool f16, int64_t outer, int64_t mid,
                                int64_t inner, const int32_t* gmap, int32_t n_groups,
                                float* absmax, uint32_t* status, cudaStream_t st) {
  const uint64_t n = (uint64_t)outer * (uint64_t)mid * (uint64_t)inner;
  if (n + 64 < (1ull << 32)) {
    const uint32_t n32 = (uint32_t)n, m32 = (uint32_t)mid, i32 = (uint32_t)inner;
    return f16 ? group_absmax_p<true, uint32_t>(src, n32, m32, i32, gmap, n_groups, absmax, status, st)
               : group_absmax_p<false, uint32_t>(src, n32, m32, i32, gmap, n_groups, absmax, status, st);
  }
  return f16 ? group_absmax_p<true, uint64_t>(src, n, (uint64_t)mid, (uint64_t)inner, gmap, n_groups,
                                              absmax, status, st)
             : group_absmax_p<false, uint64_t>(src, n, (uint64_t)mid, (uint64_t)inner, gmap,
                                               n_groups, absmax, status, st);
}

cudaError_t launch_softedge_encode(const void* src, bool f16, int64_t n, float scale, float lo,
                                   float hi, int log2_ratio, uint8_t* codes, uint32_t* status,
                                   cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const SeSteps steps = se_steps(scale, log2_ratio);
  const size_t smem32 = (size_t)acc_smem_offset<false>();
  if (f16) {
    // the table kernel: 64 KB of codes + the pipeline's stages per CTA
    const size_t smem_lut = kLutBytes + (size_t)acc_smem_offset<true>();
    const uint64_t tiles = ((uint64_t)n + stream::kTileElems - 1) / stream::kTileElems;
    uint64_t grid = (uint64_t)sm_count() * kLutCtasPerSm;
    if (grid > tiles) grid = tiles ? tiles : 1;
    auto go = [&](auto kern, auto nn) {
      cudaError_t e =
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_lut);
      if (e != cudaSuccess) return e;
      // two 113 KB CTAs per SM need the whole shared-memory carveout
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
      kern<<<(unsigned)grid, stream::kThreads, smem_lut, st>>>(
          static_cast<const uint16_t*>(src), nn, lo, hi, steps, codes, status);
      return cudaGetLastError();
    };
    if ((uint64_t)n + 64 < (1ull << 32)) return go(se_encode_lut_kernel<uint32_t>, (uint32_t)n);
    return go(se_encode_lut_kernel<uint64_t>, (uint64_t)n);
  }
  if ((uint64_t)n + 64 < (1ull << 32)) {
    const uint32_t n32 = (uint32_t)n;
    return launch_stream(se_encode_kernel<false, uint32_t>, (uint64_t)n, smem32, st, src, n32, lo,
                         hi, steps, codes, status);
  }
  const uint64_t n64 = (uint64_t)n;
  return launch_stream(se_encode_kernel<false, uint64_t>, n64, smem32, st, src, n64, lo, hi,
                       steps, codes, status);
}

cudaError_t launch_softedge_decode(const uint8_t* codes, int64_t n, float scale, int log2_ratio,
                                   float* out, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const SeSteps steps = se_steps(scale, log2_ratio);
  if ((uint64_t)n + 64 < (1ull << 32)) {
    const uint32_t n32 = (uint32_t)n;
    se_decode_kernel<uint32_t><<<grid_for(n32), kThreads, 0, st>>>(codes, n32, steps, out);
  } else {
    const uint64_t n64 = (uint64_t)n;
    se_decode_kernel<uint64_t><<<grid_for(n64), kThreads, 0, st>>>(codes, n64, steps, out);
  }
  return cudaGetLastError();
}

}  // namespace ssmq
