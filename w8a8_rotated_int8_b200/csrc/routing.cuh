// Router softmax, expert-choice top-C, row gather and the final bf16 store.
//
// "MLX Nucleus-Image", opening paragraph: 64 routed experts per layer with
// expert-choice routing; table "Conversion notes": each expert picks its
// top-C tokens and the expert outputs are scattered back to their tokens.
#pragma once

#include "common.cuh"

namespace convrot {

// ---------------------------------------------------------------- softmax --
// Per-token softmax of the router logits over E experts, evaluated in fp64 and
// rounded once to fp32, written transposed (S_t[e, t]) so each expert's
// scores are contiguous for the top-C selection. 32 tokens per CTA (one per
// warp); the [E, 32] tile goes through shared memory so the transposed store
// writes 128-byte rows. Optionally zeroes the same 32 rows of an fp32 buffer
// (the combine accumulator) to save a separate pass.
constexpr int kSmTokens = 32;

__global__ void __launch_bounds__(1024) router_softmax_kernel(
    const __nv_bfloat16* __restrict__ logits, int T, int E, float* __restrict__ S_t,
    float* __restrict__ clear, int64_t clear_cols) {
  extern __shared__ float sm_tile[];  // [E][32]
  const int t0 = blockIdx.x * kSmTokens;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned short* lg = reinterpret_cast<const unsigned short*>(logits);
  const int t = t0 + warp;  // one token per warp
  if (t < T) {
    double l[8];
    double m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      l[j] = (e < E) ? (double)__uint_as_float((uint32_t)__ldg(lg + (int64_t)t * E + e) << 16)
                     : -INFINITY;
      m = fmax(m, l[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    double ex[8];
    double sum = 0.0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      ex[j] = (e < E) ? exp(__dsub_rn(l[j], m)) : 0.0;
      sum = __dadd_rn(sum, ex[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum = __dadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < E) sm_tile[e * kSmTokens + warp] = __double2float_rn(__ddiv_rn(ex[j], sum));
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < E * kSmTokens; idx += blockDim.x) {
    const int e = idx / kSmTokens, tl = idx - e * kSmTokens;
    if (t0 + tl < T) S_t[(int64_t)e * T + t0 + tl] = sm_tile[idx];
  }
  if (clear != nullptr) {
    const int nrows = min(kSmTokens, T - t0);
    float4* base = reinterpret_cast<float4*>(clear + (int64_t)t0 * clear_cols);
    const int64_t n4 = (int64_t)nrows * clear_cols / 4;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t j = threadIdx.x; j < n4; j += blockDim.x) base[j] = z;
  }
}

// ------------------------------------------------------------------ top-C --
// Order-preserving map of an fp32 bit pattern to an unsigned key (-0 == +0).
__device__ __forceinline__ uint32_t score_key(uint32_t bits) {
  if (bits == 0x80000000u) bits = 0u;
  return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}

constexpr int kTopcThreads = 1024;

__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    uint32_t t = lane < nw ? warp_tot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    warp_tot[lane] = ti - t;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const uint32_t res = warp_tot[warp] + incl - v;
  __syncthreads();
  return res;
}

// One CTA per expert: radix-select (four 8-bit digits, most significant
// first) of the C-th largest score key, then an ordered compaction that
// takes every key above the threshold and the first k keys equal to it in
// token order. Result: the C largest scores with ties to the lower token
// index, listed in ascending token order.
// When `slot` is given it also receives, for every token t, the position c of
// t in this expert's list (slot[e, t] = c) or -1 if the expert did not pick t.
__global__ void __launch_bounds__(kTopcThreads) topc_kernel(const float* __restrict__ S_t, int T,
                                                            int C, int32_t* __restrict__ idx,
                                                            float* __restrict__ w,
                                                            int32_t* __restrict__ slot) {
  const int e = blockIdx.x;
  const uint32_t* u = reinterpret_cast<const uint32_t*>(S_t) + (int64_t)e * T;
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_digit, s_k;
  if (C <= 0) {
    if (slot != nullptr)
      for (int t = threadIdx.x; t < T; t += blockDim.x) slot[(int64_t)e * T + t] = -1;
    return;
  }
  uint32_t prefix = 0u, mask = 0u, k = (uint32_t)C;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const uint32_t key = score_key(__ldg(u + t));
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8];
      uint32_t local = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[8 * lane + j];
        local += c[j];
      }
      uint32_t incl = local;  // sum over lanes >= lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += o;
      }
      uint32_t run = incl - local;  // keys in higher digits
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        const uint32_t above = run;
        run += c[j];
        if (above < k && run >= k) {
          s_digit = (uint32_t)(8 * lane + j);
          s_k = k - above;
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    k = s_k;
    __syncthreads();
  }
  const uint32_t thr = prefix;
  const int seg = (T + blockDim.x - 1) / blockDim.x;
  const int tb = min(T, (int)threadIdx.x * seg);
  const int te = min(T, tb + seg);
  uint32_t n_eq = 0u;
  for (int t = tb; t < te; ++t) n_eq += (score_key(u[t]) == thr) ? 1u : 0u;
  const uint32_t eq_before = block_excl_scan(n_eq, warp_tot);
  uint32_t n_sel = 0u;
  {
    uint32_t seen = eq_before;
    for (int t = tb; t < te; ++t) {
      const uint32_t key = score_key(u[t]);
      if (key > thr) {
        ++n_sel;
      } else if (key == thr) {
        if (seen < k) ++n_sel;
        ++seen;
      }
    }
  }
  uint32_t pos = block_excl_scan(n_sel, warp_tot);
  {
    uint32_t seen = eq_before;
    for (int t = tb; t < te; ++t) {
      const uint32_t bits = u[t];
      const uint32_t key = score_key(bits);
      bool take = false;
      if (key > thr) {
        take = true;
      } else if (key == thr) {
        take = seen < k;
        ++seen;
      }
      int32_t my_slot = -1;
      if (take) {
        if (pos < (uint32_t)C) {
          idx[(int64_t)e * C + pos] = t;
          w[(int64_t)e * C + pos] = __uint_as_float(bits);
          my_slot = (int32_t)pos;
        } else {
          atomicOr(&g_device_error, kErrBadIndex);
        }
        ++pos;
      }
      if (slot != nullptr) slot[(int64_t)e * T + t] = my_slot;
    }
  }
}

// ----------------------------------------------------------------- gather --
// dst[r, :] = src[idx[r], :], s_dst[r] = s_src[idx[r]]; one warp per row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const int8_t* __restrict__ src,
                                                          const float* __restrict__ s_src,
                                                          int64_t n_src,
                                                          const int32_t* __restrict__ idx,
                                                          int64_t n_rows, int K,
                                                          int8_t* __restrict__ dst,
                                                          float* __restrict__ s_dst) {
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n_rows) return;
  const int t = __ldg(idx + r);
  if (t < 0 || t >= n_src) {
    if (lane == 0) atomicOr(&g_device_error, kErrBadIndex);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>(src + (int64_t)t * K);
  uint4* d = reinterpret_cast<uint4*>(dst + r * K);
  const int n16 = K >> 4;
  for (int c0 = 0; c0 < n16; c0 += 128) {
    uint4 buf[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c < n16) buf[k] = __ldg(s + c);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c < n16) d[c] = buf[k];
    }
  }
  if (lane == 0) s_dst[r] = __ldg(s_src + t);
}

// ---------------------------------------------------------------- combine --
// y[t, :] = bf16(sum over experts e = 0, 1, ..., E-1 that picked t of
// zw[e * C + slot[e, t], :]) with the sum in fp32 in that order (a token no
// expert picked gets 0). One CTA of kCombineThreads per token: the first warp
// lists the token's rows in expert order, then every thread owns up to
// kCombineQuads float4 columns and loads them for two experts at a time
// before adding, so many independent reads are in flight.
constexpr int kCombineMaxE = 256;
constexpr int kCombineThreads = 128;
constexpr int kCombineQuads = 4;  // float4 columns per thread per pass
__global__ void __launch_bounds__(kCombineThreads) combine_rows_kernel(
    const float* __restrict__ zw, const int32_t* __restrict__ slot, int E, int T, int C, int d,
    __nv_bfloat16* __restrict__ y) {
  __shared__ int32_t sel[kCombineMaxE];
  __shared__ int s_n;
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    int n = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = (e < E) ? __ldg(slot + (int64_t)e * T + t) : -1;
      const bool bad = c >= C;
      if (bad) atomicOr(&g_device_error, kErrBadIndex);
      const bool has = c >= 0 && !bad;
      const unsigned m = __ballot_sync(0xffffffffu, has);
      if (has) sel[n + __popc(m & ((1u << lane) - 1u))] = e * C + c;
      n += __popc(m);
    }
    if (lane == 0) s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  const int d4 = d >> 2;
  uint2* yrow = reinterpret_cast<uint2*>(y + (int64_t)t * d);
  for (int q0 = threadIdx.x; q0 < d4; q0 += kCombineThreads * kCombineQuads) {
    float4 acc[kCombineQuads];
#pragma unroll
    for (int u = 0; u < kCombineQuads; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    int k = 0;
    for (; k + 2 <= n; k += 2) {
      const float4* r0 = reinterpret_cast<const float4*>(zw + (int64_t)sel[k] * d);
      const float4* r1 = reinterpret_cast<const float4*>(zw + (int64_t)sel[k + 1] * d);
      float4 a[kCombineQuads], b[kCombineQuads];
#pragma unroll
      for (int u = 0; u < kCombineQuads; ++u) {
        const int q = q0 + u * kCombineThreads;
        if (q < d4) {
          a[u] = __ldcs(r0 + q);
          b[u] = __ldcs(r1 + q);
        }
      }
#pragma unroll
      for (int u = 0; u < kCombineQuads; ++u) {
        acc[u].x = __fadd_rn(__fadd_rn(acc[u].x, a[u].x), b[u].x);
        acc[u].y = __fadd_rn(__fadd_rn(acc[u].y, a[u].y), b[u].y);
        acc[u].z = __fadd_rn(__fadd_rn(acc[u].z, a[u].z), b[u].z);
        acc[u].w = __fadd_rn(__fadd_rn(acc[u].w, a[u].w), b[u].w);
      }
    }
    if (k < n) {
      const float4* r0 = reinterpret_cast<const float4*>(zw + (int64_t)sel[k] * d);
#pragma unroll
      for (int u = 0; u < kCombineQuads; ++u) {
        const int q = q0 + u * kCombineThreads;
        if (q < d4) {
          const float4 a = __ldcs(r0 + q);
          acc[u].x = __fadd_rn(acc[u].x, a.x);
          acc[u].y = __fadd_rn(acc[u].y, a.y);
          acc[u].z = __fadd_rn(acc[u].z, a.z);
          acc[u].w = __fadd_rn(acc[u].w, a.w);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kCombineQuads; ++u) {
      const int q = q0 + u * kCombineThreads;
      if (q < d4) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t*>(&lo);
        o.y = *reinterpret_cast<const uint32_t*>(&hi);
        yrow[q] = o;
      }
    }
  }
}

// ---------------------------------------------------------------- convert --
// y = bf16_rne(x), four elements per thread iteration.
__device__ __forceinline__ uint2 bf16x4(float4 f) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(f.x, f.y);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(f.z, f.w);
  uint2 o;
  o.x = *reinterpret_cast<const uint32_t*>(&lo);
  o.y = *reinterpret_cast<const uint32_t*>(&hi);
  return o;
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ x, int64_t n4,
                                                          __nv_bfloat16* __restrict__ y) {
  const float4* x4 = reinterpret_cast<const float4*>(x);
  uint2* y2 = reinterpret_cast<uint2*>(y);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n4; i += 4 * stride) {
    const float4 a = __ldcs(x4 + i), b = __ldcs(x4 + i + stride);
    const float4 c = __ldcs(x4 + i + 2 * stride), d = __ldcs(x4 + i + 3 * stride);
    y2[i] = bf16x4(a);
    y2[i + stride] = bf16x4(b);
    y2[i + 2 * stride] = bf16x4(c);
    y2[i + 3 * stride] = bf16x4(d);
  }
  for (; i < n4; i += stride) y2[i] = bf16x4(__ldcs(x4 + i));
}

// --------------------------------------------------------- wait self-test --
// Waits on an mbarrier that nothing arrives on, with the given limit, through
// the same bounded wait the GEMM pipeline uses; it must give up, record
// kErrSelfTest and return.
__global__ void wait_selftest_kernel(unsigned long long limit_ns, int* result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait_limit(&bar, 0, &abort_flag, kErrSelfTest, limit_ns);
    *result = ok ? 1 : 0;
  }
}

}  // namespace convrot
