// append.cuh -- writing new tokens into the absorb path's latent caches.
//
// "Naive vs Absorb Attention Implementations in DeepSeek-V3", section "Absorb
// Implementation Cache Design": per token the absorb path caches the compressed
// key-value vector (kv_cache, kv_lora_rank values) and the rotary key (pe_cache,
// qk_rope_head_dim values).  "Latent KV expansion with split" states that the
// compressed KV is RMS-normalised.  For new token n:
//   kv_cache[slot[n]] = kv_new[n] / sqrt(mean(kv_new[n]^2) + eps) * gamma
//   pe_cache[slot[n]] = k_pe_new[n] with pair (2i, 2i+1) turned by
//                       position[n] * base^(-2i/R)
// One warp per two tokens, every load issued before any arithmetic (the op is a
// pure stream of 2 x (C + R) elements per token, bound by the bytes each SM keeps
// in flight): 16-byte loads and stores of the latent rows (a warp covers 512
// contiguous bytes per instruction), the sums of squares reduced by shuffles,
// one lane per rotary pair.  The rotation angle is formed and reduced modulo 2 pi
// in double precision (positions reach 10^5 and beyond, where a float product
// loses the angle); CUDA's sincosf then takes the reduced angle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {
namespace append {

constexpr int kWarpsPerBlock = 4;

template <typename T> struct Vec;   // 16-byte vector of T <-> 8 or 4 floats
template <> struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void unpack(const uint4& v, float* f) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  }
  __device__ static uint4 pack(const float* f) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      u[i] = *reinterpret_cast<const uint32_t*>(&p);
    }
    return make_uint4(u[0], u[1], u[2], u[3]);
  }
};
template <> struct Vec<float> {
  static constexpr int kN = 4;
  __device__ static void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y); f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

// C is a multiple of 8 (bf16) or 4 (fp32) and at most kMaxC; R is even and at most 2 * 32 * kMaxPairsPerLane.
constexpr int kMaxC = 1024;
constexpr int kMaxPairsPerLane = 2;

constexpr int kTokensPerWarp = 2;   // more loads in flight per warp: the op is latency-bound per SM

// PER_LANE: 16-byte vectors of a latent row per lane (C / (32 * 16-byte vector elements), rounded up).
template <typename T, int PER_LANE>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    append_kernel(const T* __restrict__ kv_new, const T* __restrict__ pe_new, const T* __restrict__ gamma, float eps,
                  double log2_base, const int32_t* __restrict__ positions, const int64_t* __restrict__ slots,
                  int64_t n_tokens, int C, int R, T* __restrict__ kv_cache, T* __restrict__ pe_cache,
                  int64_t cache_rows) {
  using V = Vec<T>;
  constexpr int kPerLane = PER_LANE;
  const int64_t n0 = ((int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5)) * kTokensPerWarp;
  if (n0 >= n_tokens) return;   // warp-uniform
  const int lane = (int)(threadIdx.x & 31);
  const int nvec = C / V::kN;

  // every load of the warp's tokens first
  int64_t slot[kTokensPerWarp];
  double pos[kTokensPerWarp];
  uint4 x[kTokensPerWarp][kPerLane];   // raw 16-byte vectors, unpacked when used (fewer live registers)
  float pa[kTokensPerWarp][kMaxPairsPerLane], pb[kTokensPerWarp][kMaxPairsPerLane];
#pragma unroll
  for (int t = 0; t < kTokensPerWarp; ++t) {
    const int64_t n = n0 + t;
    const bool valid = n < n_tokens;
    slot[t] = valid ? __ldg(slots + n) : -1;
    pos[t] = valid ? (double)__ldg(positions + n) : 0.0;
    const uint4* src = reinterpret_cast<const uint4*>(kv_new + n * C);
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) {
      const int v = lane + 32 * k;
      if (valid && v < nvec) x[t][k] = __ldg(src + v);
    }
#pragma unroll
    for (int k = 0; k < kMaxPairsPerLane; ++k) {
      const int i = lane + 32 * k;
      if (valid && 2 * i < R) {
        pa[t][k] = Elem<T>::load(pe_new + n * R + 2 * i);
        pb[t][k] = Elem<T>::load(pe_new + n * R + 2 * i + 1);
      }
    }
  }
  const uint4* gv = reinterpret_cast<const uint4*>(gamma);

#pragma unroll
  for (int t = 0; t < kTokensPerWarp; ++t) {
    if (n0 + t >= n_tokens) break;   // warp-uniform
    // latent row: sum of squares, scale, store
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kPerLane; ++k)
      if (lane + 32 * k < nvec) {
        float f[V::kN];
        V::unpack(x[t][k], f);
#pragma unroll
        for (int i = 0; i < V::kN; ++i) ss = fmaf(f[i], f[i], ss);
      }
    ss = warp_sum(ss);
    if (slot[t] < 0 || slot[t] >= cache_rows) continue;   // outside the cache: nothing is written
    const float inv = rsqrtf(ss / (float)C + eps);
    uint4* dst = reinterpret_cast<uint4*>(kv_cache + slot[t] * C);
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) {
      const int v = lane + 32 * k;
      if (v < nvec) {
        float g[V::kN];
        if (gamma) V::unpack(__ldg(gv + v), g);
        float y[V::kN];
        V::unpack(x[t][k], y);
#pragma unroll
        for (int i = 0; i < V::kN; ++i) y[i] = y[i] * inv * (gamma ? g[i] : 1.f);
        dst[v] = V::pack(y);
      }
    }
    // rotary key: lane turns pairs lane, lane + 32.  The angle is formed and reduced to
    // [-pi, pi] in double precision, then its sine and cosine are taken in float.
#pragma unroll
    for (int k = 0; k < kMaxPairsPerLane; ++k) {
      const int i = lane + 32 * k;
      if (2 * i < R) {
        const double theta = pos[t] * exp2(-2.0 * i / R * log2_base);
        const double two_pi = 6.283185307179586476925286766559;
        const float r = (float)(theta - two_pi * rint(theta / two_pi));
        float sf, cf;
        sincosf(r, &sf, &cf);
        const float a = pa[t][k], b = pb[t][k];
        Elem<T>::store(pe_cache + slot[t] * R + 2 * i, a * cf - b * sf);
        Elem<T>::store(pe_cache + slot[t] * R + 2 * i + 1, a * sf + b * cf);
      }
    }
  }
  // The rows are visible device-wide before this thread exits: an attention call launched next
  // starts its cache stream before it waits for this kernel's completion.
  __threadfence();
}

}  // namespace append
}  // namespace mla
