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
// warp, NJ = ceil(E / 32) experts per lane, so no lane evaluates an exp for
// an expert that does not exist); the [E, 32] tile goes through shared memory
// so the transposed store writes 128-byte rows.
constexpr int kSmTokens = 32;

template <int NJ>
__global__ void __launch_bounds__(1024) router_softmax_kernel(
    const __nv_bfloat16* __restrict__ logits, int T, int E, float* __restrict__ S_t) {
  extern __shared__ float sm_tile[];  // [E][32]
  const int t0 = blockIdx.x * kSmTokens;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned short* lg = reinterpret_cast<const unsigned short*>(logits);
  const int t = t0 + warp;  // one token per warp
  if (t < T) {
    double l[NJ];
    double m = -INFINITY;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = lane + 32 * j;
      l[j] = (e < E) ? (double)__uint_as_float((uint32_t)__ldg(lg + (int64_t)t * E + e) << 16)
                     : -INFINITY;
      m = fmax(m, l[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    double ex[NJ];
    double sum = 0.0;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = lane + 32 * j;
      ex[j] = 0.0;
      if (e < E) ex[j] = exp(__dsub_rn(l[j], m));
      sum = __dadd_rn(sum, ex[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum = __dadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = lane + 32 * j;
      if (e < E) sm_tile[e * kSmTokens + warp] = __double2float_rn(__ddiv_rn(ex[j], sum));
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < E * kSmTokens; idx += blockDim.x) {
    const int e = idx / kSmTokens, tl = idx - e * kSmTokens;
    if (t0 + tl < T) S_t[(int64_t)e * T + t0 + tl] = sm_tile[idx];
  }
}

// ------------------------------------------------------------------ top-C --
// Order-preserving map of an fp32 bit pattern to an unsigned key (-0 == +0).
__device__ __forceinline__ uint32_t score_key(uint32_t bits) {
  if (bits == 0x80000000u) bits = 0u;
  return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}

// Inverse of score_key (a -0 score comes back as +0; softmax scores are >= +0).
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
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

// Register-resident top-C for T <= kTopcThreads * KPT: the same selection as
// topc_kernel (radix select of the C-th largest key, four 8-bit digits, then
// an ordered compaction), with every score read once into registers. Thread
// i owns the KPT consecutive tokens [i * KPT, i * KPT + KPT). The digit
// histograms are replicated per lane ([bin][lane] words), so the 32 lanes of
// a warp always hit 32 different banks even when they all count the same
// digit (softmax scores share their leading bits). One scan of packed
// (greater, equal) counts places every pick: a token's list position is
// (keys above the threshold before it) + min(equal keys before it, k).
template <int KPT>
__global__ void __launch_bounds__(kTopcThreads) topc_reg_kernel(const float* __restrict__ S_t,
                                                                int T, int C,
                                                                int32_t* __restrict__ idx,
                                                                float* __restrict__ w,
                                                                int32_t* __restrict__ slot) {
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* row = S_t + (int64_t)e * T;
  __shared__ uint32_t hist[256 * 32];
  __shared__ uint32_t tot[256];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_digit, s_k;
  const int t0 = threadIdx.x * KPT;
  if (C <= 0) {
    if (slot != nullptr)
      for (int t = threadIdx.x; t < T; t += blockDim.x) slot[(int64_t)e * T + t] = -1;
    return;
  }
  uint32_t key[KPT];
  if (KPT >= 4 && (T & 3) == 0 && t0 + KPT <= T) {
#pragma unroll
    for (int j = 0; j < KPT; j += 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + t0 + j));
      key[j] = score_key(v.x);
      key[j + 1] = score_key(v.y);
      key[j + 2] = score_key(v.z);
      key[j + 3] = score_key(v.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      key[j] = (t0 + j < T) ? score_key(__float_as_uint(__ldg(row + t0 + j))) : 0u;
  }
  const int n_valid = max(0, min(KPT, T - t0));

  uint32_t prefix = 0u, mask = 0u, k = (uint32_t)C;
  for (int shift = 24; shift >= 0; shift -= 8) {
    uint4* h4 = reinterpret_cast<uint4*>(hist);
    for (int i = threadIdx.x; i < 256 * 32 / 4; i += blockDim.x) h4[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (j < n_valid && (key[j] & mask) == prefix)
        atomicAdd(&hist[((key[j] >> shift) & 255u) * 32 + lane], 1u);
    __syncthreads();
    // bin totals: warp w sums bins 8w .. 8w+7 over the 32 lane copies
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int bin = warp * 8 + b;
      const uint32_t v = __reduce_add_sync(0xffffffffu, hist[bin * 32 + lane]);
      if (lane == 0) tot[bin] = v;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8];
      uint32_t local = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = tot[8 * lane + j];
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
  }
  const uint32_t thr = prefix;
  uint32_t n_gt = 0u, n_eq = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if (j < n_valid) {
      n_gt += key[j] > thr ? 1u : 0u;
      n_eq += key[j] == thr ? 1u : 0u;
    }
  }
  // counts stay below 2^16 (T <= 16384): one scan of both
  const uint32_t before = block_excl_scan((n_gt << 16) | n_eq, warp_tot);
  uint32_t gt_seen = before >> 16, eq_seen = before & 0xffffu;
  int32_t my_slot[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    my_slot[j] = -1;
    if (j < n_valid) {
      const bool gt = key[j] > thr, eq = key[j] == thr;
      if (gt || (eq && eq_seen < k)) {
        const uint32_t pos = gt_seen + min(eq_seen, k);
        if (pos < (uint32_t)C) {
          idx[(int64_t)e * C + pos] = t0 + j;
          w[(int64_t)e * C + pos] = key_score(key[j]);
          my_slot[j] = (int32_t)pos;
        } else {
          atomicOr(&g_device_error, kErrBadIndex);
        }
      }
      gt_seen += gt ? 1u : 0u;
      eq_seen += eq ? 1u : 0u;
    }
  }
  if (slot != nullptr) {
    int32_t* srow = slot + (int64_t)e * T;
    if (KPT >= 4 && (T & 3) == 0 && t0 + KPT <= T) {
#pragma unroll
      for (int j = 0; j < KPT; j += 4)
        *reinterpret_cast<int4*>(srow + t0 + j) =
            make_int4(my_slot[j], my_slot[j + 1], my_slot[j + 2], my_slot[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < KPT; ++j)
        if (j < n_valid) srow[t0 + j] = my_slot[j];
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
// y[t, :] = bf16(sum over experts e = 0, 1, ..., E-1 that picked t, with
// c = slot[e, t], of fp32(s_t[e, t] * z[e*C + c, :])): every product rounded
// to fp32, the sum in fp32 in that order (a token no expert picked gets 0).
// z holds the experts' BF16 outputs; s_t[e, t] is the router score of token t
// for expert e, i.e. the weight top-C stored for the pick, so the slot and
// weight look-ups are independent loads.
//
// One CTA of kCombineThreads per token. Every warp builds the token's list
// (rows and weights in ascending expert order) itself from one round of
// loads, so no CTA-wide barrier is needed; then each thread sums its
// 8-column (16-byte) vectors over the rows, two rows' loads in flight at a
// time.
constexpr int kCombineThreads = 128;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombineVecs = 2;  // 8-column vectors per thread per pass

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

template <int NJ>
__global__ void __launch_bounds__(kCombineThreads) combine_rows_kernel(
    const __nv_bfloat16* __restrict__ z, const float* __restrict__ s_t,
    const int32_t* __restrict__ slot, int E, int T, int C, int d, __nv_bfloat16* __restrict__ y) {
  __shared__ int32_t sel_all[kCombineWarps][32 * NJ];
  __shared__ float sw_all[kCombineWarps][32 * NJ];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* sel = sel_all[warp];
  float* sw = sw_all[warp];
  int32_t sv[NJ];
  float wv[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    sv[j] = e < E ? __ldg(slot + (int64_t)e * T + t) : -1;
    wv[j] = e < E ? __ldg(s_t + (int64_t)e * T + t) : 0.0f;
  }
  int n = 0;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const bool bad = sv[j] >= C;
    if (bad && warp == 0) atomicOr(&g_device_error, kErrBadIndex);
    const bool has = sv[j] >= 0 && !bad;
    const unsigned m = __ballot_sync(0xffffffffu, has);
    if (has) {
      const int pos = n + __popc(m & ((1u << lane) - 1u));
      sel[pos] = (lane + 32 * j) * C + sv[j];
      sw[pos] = wv[j];
    }
    n += __popc(m);
  }
  __syncwarp();
  const int d8 = d >> 3;
  uint4* yrow = reinterpret_cast<uint4*>(y + (int64_t)t * d);
  for (int q0 = threadIdx.x; q0 < d8; q0 += kCombineThreads * kCombineVecs) {
    float acc[kCombineVecs][8];
#pragma unroll
    for (int u = 0; u < kCombineVecs; ++u)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
    int k = 0;
    for (; k + 2 <= n; k += 2) {
      const uint4* r0 = reinterpret_cast<const uint4*>(z + (int64_t)sel[k] * d);
      const uint4* r1 = reinterpret_cast<const uint4*>(z + (int64_t)sel[k + 1] * d);
      const float w0 = sw[k], w1 = sw[k + 1];
      uint4 a[kCombineVecs], b[kCombineVecs];
#pragma unroll
      for (int u = 0; u < kCombineVecs; ++u) {
        const int q = q0 + u * kCombineThreads;
        if (q < d8) {
          a[u] = __ldcs(r0 + q);
          b[u] = __ldcs(r1 + q);
        }
      }
#pragma unroll
      for (int u = 0; u < kCombineVecs; ++u) {
        if (q0 + u * kCombineThreads < d8) {
          float fa[8], fb[8];
          bf16x8_to_f32(a[u], fa);
          bf16x8_to_f32(b[u], fb);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[u][i] = __fadd_rn(__fadd_rn(acc[u][i], __fmul_rn(w0, fa[i])), __fmul_rn(w1, fb[i]));
        }
      }
    }
    if (k < n) {
      const uint4* r0 = reinterpret_cast<const uint4*>(z + (int64_t)sel[k] * d);
      const float w0 = sw[k];
#pragma unroll
      for (int u = 0; u < kCombineVecs; ++u) {
        const int q = q0 + u * kCombineThreads;
        if (q < d8) {
          float fa[8];
          bf16x8_to_f32(__ldcs(r0 + q), fa);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[u][i] = __fadd_rn(acc[u][i], __fmul_rn(w0, fa[i]));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kCombineVecs; ++u) {
      const int q = q0 + u * kCombineThreads;
      if (q < d8) {
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 pr = __floats2bfloat162_rn(acc[u][2 * i], acc[u][2 * i + 1]);
          o[i] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        yrow[q] = make_uint4(o[0], o[1], o[2], o[3]);
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
