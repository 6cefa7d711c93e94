// Bulk-copy pipeline for the streaming (HBM-bound) kernels.
//
// One producer warp keeps kStages tiles of the input in flight with the
// Blackwell bulk-copy engine (cp.async.bulk global -> shared, completion
// counted in bytes on an mbarrier); eight consumer warps turn each tile into
// outputs that they store straight to global memory with 16-byte stores.
// Tile j of a CTA is global tile blockIdx.x + j * gridDim.x and lives in stage
// j % kStages; "full" barriers signal landed bytes, "empty" barriers (one
// arrival per consumer warp) hand a stage back to the producer.  Every wait
// is bounded: on giving up the waiter raises SSMQ_DEV_TIMEOUT, the CTA stops
// taking tiles, and the producer waits (bounded) for its copies in flight
// before the CTA exits.  The partial last tile is read with plain loads by
// the CTA that would own it.
#pragma once

#include <stdlib.h>

#include "common.cuh"
#include "tc.cuh"

namespace ssmq {
namespace stream {

constexpr int kVec = 16;                       // elements per consumer thread per tile
constexpr int kConsumers = 256;                // 8 consumer warps
constexpr int kThreads = kConsumers + 32;      // + 1 producer warp
constexpr int kTileElems = kConsumers * kVec;  // 4096
constexpr int kInFlightBytes = 48 * 1024;      // per CTA
constexpr int kCtasPerSm = 3;
constexpr uint32_t kWaitLimit = 1u << 20;      // mbarrier probes (~1 us each)

template <int kEsz>
struct Cfg {
  static constexpr int kTileBytes = kTileElems * kEsz;
  static constexpr int kStages = kInFlightBytes / kTileBytes;
  // stage buffers, then 2 * kStages mbarriers, then the abort word
  static constexpr int kBarOff = kStages * kTileBytes;
  static constexpr int kSmem = kBarOff + 2 * kStages * 8 + 16;
};

__device__ __forceinline__ void expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc::smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}
// global -> shared bulk copy; both addresses 16-byte aligned, bytes % 16 == 0
__device__ __forceinline__ void bulk_g2s(void* sdst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          tc::smem_u32(sdst)),
      "l"(gsrc), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}

// Thread `tid`'s 16 elements of a tile in shared memory, as fp32.  The 16-byte
// pieces of a thread's vector are read in a lane-dependent order chosen so
// that every 8 consecutive lanes of one load instruction hit the 8 different
// 16-byte bank groups of a 128-byte row (4 wavefronts per warp, the minimum).
template <bool kF16>
__device__ __forceinline__ void smem16(const uint8_t* tile, int tid, float (&v)[kVec]) {
  if (kF16) {
    // lane t holds pieces 2t, 2t+1: lanes t and t+4 share a bank group
    const uint4* p = reinterpret_cast<const uint4*>(tile) + 2 * tid;
    const int f = (tid >> 2) & 1;
    const uint4 a = p[f], b = p[f ^ 1];
    const uint4 lo = f ? b : a, hi = f ? a : b;
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      v[2 * i] = x.x;
      v[2 * i + 1] = x.y;
    }
  } else {
    // lane t holds pieces 4t .. 4t+3 (bank groups 4 (t & 1) + k); lanes with
    // bit 1 set read their pieces in the order k ^ 2, which halves the
    // conflicts (8 wavefronts per warp instead of 16) with static registers
    const float4* p = reinterpret_cast<const float4*>(tile) + 4 * tid;
    const bool sw = (tid & 2) != 0;
    float4 q[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) q[k] = p[sw ? k ^ 2 : k];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 x = sw ? q[k ^ 2] : q[k];
      v[4 * k] = x.x;
      v[4 * k + 1] = x.y;
      v[4 * k + 2] = x.z;
      v[4 * k + 3] = x.w;
    }
  }
}

// Thread `tid`'s 16 binary16 elements of a tile as 8 words of raw bits
// (element 2 i in the low half of w[i]), same bank-conflict-free order as
// smem16.
__device__ __forceinline__ void smem16_bits(const uint8_t* tile, int tid, uint32_t (&w)[8]) {
  const uint4* p = reinterpret_cast<const uint4*>(tile) + 2 * tid;
  const int f = (tid >> 2) & 1;
  const uint4 a = p[f], b = p[f ^ 1];
  const uint4 lo = f ? b : a, hi = f ? a : b;
  w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
  w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
}

template <bool kF16, typename Idx>
__device__ __forceinline__ void global16(const void* src, Idx e0, float (&v)[kVec]) {
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
__device__ __forceinline__ float global1(const void* src, Idx e) {
  if (kF16) return h2f(static_cast<const uint16_t*>(src)[e]);
  return static_cast<const float*>(src)[e];
}

struct NoPrologue {
  __device__ __forceinline__ void operator()() const {}
};

// Runs the pipeline over src[0, n) as CTA c of G working on it (tile j of
// the CTA is tile c + j G).  Every thread of the CTA (kThreads) must call it.
// vec(x, e0) consumes the 16 elements e0..e0+15; one(v, e) a single element
// of the ragged end.  prologue() runs on the consumer threads before their
// first tile, while the producer's first copies are in flight, and is
// followed by a barrier of the consumers.  Returns with every copy of this
// CTA complete.
// kBits (binary16 sources only): vec receives the raw bits, vec(const
// uint32_t (&w)[8], e0), instead of fp32 values.
template <bool kF16, typename Idx, class Vec, class One, class Pro = NoPrologue,
          bool kBits = false>
__device__ __forceinline__ void run_part(const void* __restrict__ src, Idx n, uint8_t* smem,
                                         const Idx c, const Idx G, Vec&& vec, One&& one,
                                         uint32_t& flags, uint32_t limit = kWaitLimit,
                                         Pro&& prologue = Pro()) {
  constexpr int kEsz = kF16 ? 2 : 4;
  using C = Cfg<kEsz>;
  constexpr int S = C::kStages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + S;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(empty + S);
  const int tid = threadIdx.x;
  const Idx ntiles = n / (Idx)kTileElems;
  const Idx J = c < ntiles ? (ntiles - c + G - 1) / G : 0;  // full tiles of this CTA

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, kConsumers / 32);
    }
    *abort_flag = 0u;
  }
  __syncthreads();

  Idx issued = 0;  // copies issued (producer lane)
  if (tid >= kConsumers) {
    // ---- producer warp: lane 0 issues the copies
    if (tid == kConsumers) {
      for (Idx j = 0; j < J; ++j) {
        const int s = (int)(j % S);
        if (j >= (Idx)S) {
          const uint32_t par = (uint32_t)((j / S - 1) & 1);
          bool ok = false;
          for (uint32_t i = 0; i < limit && !ok; ++i) {
            ok = tc::mbar_try(empty + s, par);
            if (!ok && *abort_flag) break;
          }
          if (!ok) {
            if (!*abort_flag) flags |= SSMQ_DEV_TIMEOUT;
            *abort_flag = 1u;
            break;
          }
        }
        const Idx tile = c + j * G;
        expect_tx(full + s, (uint32_t)C::kTileBytes);
        bulk_g2s(smem + s * C::kTileBytes,
                 static_cast<const uint8_t*>(src) + (uint64_t)tile * C::kTileBytes,
                 (uint32_t)C::kTileBytes, full + s);
        issued = j + 1;
      }
    }
    __syncwarp();
  } else {
    // ---- consumers
    prologue();
    tc::named_sync(1, kConsumers);
    const int lane = tid & 31;
    for (Idx j = 0; j < J; ++j) {
      const int s = (int)(j % S);
      const uint32_t par = (uint32_t)((j / S) & 1);
      bool ok = false;
      for (uint32_t i = 0; i < limit && !ok; ++i) {
        ok = tc::mbar_try(full + s, par);
        if (!ok && *abort_flag) break;
      }
      ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
      if (!ok) {
        if (!*abort_flag) flags |= SSMQ_DEV_TIMEOUT;
        *abort_flag = 1u;
        break;
      }
      const Idx tile = c + j * G;
      if constexpr (kBits) {
        static_assert(kF16, "raw bits are binary16 only");
        uint32_t w[8];
        smem16_bits(smem + s * C::kTileBytes, tid, w);
        vec(w, tile * (Idx)kTileElems + (Idx)tid * kVec);
      } else {
        float x[kVec];
        smem16<kF16>(smem + s * C::kTileBytes, tid, x);
        vec(x, tile * (Idx)kTileElems + (Idx)tid * kVec);
      }
      __syncwarp();
      if (lane == 0) arrive(empty + s);
    }
    // the ragged last tile, with plain loads
    if (ntiles % G == c && !*abort_flag) {
      for (Idx e0 = ntiles * (Idx)kTileElems + (Idx)tid * kVec; e0 < n; e0 += (Idx)kConsumers * kVec) {
        if (e0 + kVec <= n) {
          if constexpr (kBits) {
            const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + e0);
            const uint4 a = __ldg(p), b = __ldg(p + 1);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            vec(w, e0);
          } else {
            float x[kVec];
            global16<kF16, Idx>(src, e0, x);
            vec(x, e0);
          }
        } else {
          for (Idx e = e0; e < n; ++e) one(global1<kF16, Idx>(src, e), e);
        }
      }
    }
  }
  __syncthreads();
  if (tid == kConsumers && *abort_flag) {
    // a wait gave up: every copy issued lands before the CTA may exit (the
    // last kStages issued are the only ones that can still be in flight)
    for (Idx j = issued > (Idx)S ? issued - S : 0; j < issued; ++j)
      if (!tc::mbar_wait(full + (int)(j % S), (uint32_t)((j / S) & 1), kWaitLimit))
        flags |= SSMQ_DEV_TIMEOUT;
  }
}

// The whole grid on src[0, n).
template <bool kF16, typename Idx, class Vec, class One>
__device__ __forceinline__ void run(const void* __restrict__ src, Idx n, uint8_t* smem, Vec&& vec,
                                    One&& one, uint32_t& flags, uint32_t limit = kWaitLimit) {
  run_part<kF16, Idx>(src, n, smem, (Idx)blockIdx.x, (Idx)gridDim.x, vec, one, flags, limit);
}

// Probes before a pipeline wait (a consumer waiting for a tile, the producer
// for a free stage) gives up: kWaitLimit, unless the environment variable
// SSMQ_WAIT_LIMIT asks for fewer -- the tests of the timeout path set 0, so
// that every such wait gives up at once, SSMQ_DEV_TIMEOUT is raised and the
// CTAs return.  The drain of copies already in flight always keeps the full
// limit, so no copy lands after its CTA has exited.
inline uint32_t wait_limit() {
  const char* v = getenv("SSMQ_WAIT_LIMIT");
  if (!v || !*v) return kWaitLimit;
  char* end = nullptr;
  const unsigned long x = strtoul(v, &end, 10);
  return (end && *end == '\0' && x < kWaitLimit) ? (uint32_t)x : kWaitLimit;
}

template <int kEsz>
constexpr int smem_bytes() {
  return Cfg<kEsz>::kSmem;
}

// persistent grid: kCtasPerSm CTAs per SM, never more than the tiles (one
// CTA at least, for the ragged tail)
inline unsigned grid_for(uint64_t n, int sms) {
  const uint64_t tiles = (n + kTileElems - 1) / kTileElems;
  uint64_t g = (uint64_t)sms * kCtasPerSm;
  if (g > tiles) g = tiles;
  return (unsigned)(g ? g : 1);
}

}  // namespace stream
}  // namespace ssmq
