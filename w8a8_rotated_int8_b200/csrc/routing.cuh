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
// scores are contiguous for the top-C selection. kSmTokens tokens per CTA
// (one per warp, NJ = ceil(E / 32) experts per lane, so no lane evaluates an
// exp for an expert that does not exist); the [E, kSmTokens] tile goes
// through shared memory so the transposed store writes whole 32-byte
// sectors. Eight tokens per CTA spread even T = 2048 over every SM (measured
// faster than 32 tokens per CTA at T = 2048 and 8192).
constexpr int kSmTokens = 8;

template <int NJ>
__global__ void __launch_bounds__(1024) router_softmax_kernel(
    const __nv_bfloat16* __restrict__ logits, int T, int E, float* __restrict__ S_t) {
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ float sm_tile[];  // [E][kSmTokens]
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
  griddep_launch_dependents();
  griddep_wait();
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
  griddep_launch_dependents();
  griddep_wait();
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
// Also clears `zero` [n_zero] words (the synchronisation scratch of the GEMM
// that reads dst next), if given.
__global__ void __launch_bounds__(256) gather_rows_kernel(const int8_t* __restrict__ src,
                                                          const float* __restrict__ s_src,
                                                          int64_t n_src,
                                                          const int32_t* __restrict__ idx,
                                                          int64_t n_rows, int K,
                                                          int8_t* __restrict__ dst,
                                                          float* __restrict__ s_dst,
                                                          uint32_t* __restrict__ zero,
                                                          int64_t n_zero) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n_rows) return;
  if (zero != nullptr && lane == 0)
    for (int64_t i = r; i < n_zero; i += n_rows) zero[i] = 0u;
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
__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

// One CTA per run of `tpc` consecutive tokens. The [E, tpc] tiles of slots and
// router scores are read with coalesced loads (tpc consecutive tokens of one
// expert are contiguous), the picks of all tpc tokens are laid out as one
// flat list in shared memory (token by token, each in ascending expert
// order), and every thread streams its 16-byte column vector of the listed
// rows, four loads in flight, closing a token's bf16 output when the list
// moves on to the next token. Tokens without picks get 0. Launched after the
// down GEMM with programmatic dependent launch, it builds the lists (from
// slots and scores completed before that chain began) before waiting for the
// GEMM, so the list building overlaps the GEMM's tail. (Measured on B200:
// more loads in flight per thread, larger token runs, or a shared-memory
// ring fed by bulk copies were all slower; the kernel is bound by the
// latency of its dependent phases, and small runs keep more CTAs resident.)
constexpr int kCombThreads = 256;
constexpr int kCombBatch = 4;

__device__ __forceinline__ uint4 f32x8_to_bf16x8(const float (&a)[8]) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 pr = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
    o[i] = *reinterpret_cast<const uint32_t*>(&pr);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// shared memory: E * (tpc + 1) int32 slots and as many fp32 scores (stride
// tpc + 1 so a warp reading one token's column hits distinct banks), then the
// flat list: E * tpc rows (int32), weights (fp32) and token indices (uint8),
// then tpc + 1 list starts.
__host__ __device__ inline size_t combine_tokens_smem(int E, int tpc) {
  return (size_t)E * (tpc + 1) * 8 + (size_t)E * tpc * 9 + (size_t)(tpc + 1) * 4 + 64;
}

template <int NJ>
__global__ void __launch_bounds__(kCombThreads) combine_tokens_kernel(
    const __nv_bfloat16* __restrict__ z, const float* __restrict__ s_t,
    const int32_t* __restrict__ slot, int E, int T, int C, int d, int tpc,
    __nv_bfloat16* __restrict__ y) {
  griddep_launch_dependents();
  extern __shared__ __align__(16) uint8_t cm_smem[];
  const int ld = tpc + 1;
  int32_t* sl = reinterpret_cast<int32_t*>(cm_smem);
  float* sw = reinterpret_cast<float*>(sl + (size_t)E * ld);
  int32_t* fr = reinterpret_cast<int32_t*>(sw + (size_t)E * ld);
  float* fw = reinterpret_cast<float*>(fr + (size_t)E * tpc);
  int32_t* start = reinterpret_cast<int32_t*>(fw + (size_t)E * tpc);
  uint8_t* ftok = reinterpret_cast<uint8_t*>(start + tpc + 1);
  const int t0 = blockIdx.x * tpc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kCombThreads / 32;

  // 1. the [E, tpc] slot and score tiles (coalesced along the tokens)
  for (int i = threadIdx.x; i < E * tpc; i += kCombThreads) {
    const int e = i / tpc, j = i - e * tpc;
    const int t = t0 + j;
    int32_t sv = -1;
    float wv = 0.0f;
    if (t < T) {
      sv = __ldg(slot + (int64_t)e * T + t);
      wv = __ldg(s_t + (int64_t)e * T + t);
      if (sv >= C) {
        atomicOr(&g_device_error, kErrBadIndex);
        sv = -1;
      }
    }
    sl[e * ld + j] = sv;
    sw[e * ld + j] = wv;
  }
  __syncthreads();
  // 2. picks per token (warp w counts tokens w, w + 8, ...)
  for (int j = warp; j < tpc; j += nwarps) {
    int n = 0;
#pragma unroll
    for (int k = 0; k < NJ; ++k) {
      const int e = lane + 32 * k;
      n += __popc(__ballot_sync(0xffffffffu, e < E && sl[e * ld + j] >= 0));
    }
    if (lane == 0) start[j + 1] = n;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    start[0] = 0;
    for (int j = 0; j < tpc; ++j) start[j + 1] += start[j];
  }
  __syncthreads();
  // 3. the flat list, each token's picks in ascending expert order
  for (int j = warp; j < tpc; j += nwarps) {
    int pos = start[j];
#pragma unroll
    for (int k = 0; k < NJ; ++k) {
      const int e = lane + 32 * k;
      const int32_t sv = e < E ? sl[e * ld + j] : -1;
      const unsigned m = __ballot_sync(0xffffffffu, sv >= 0);
      if (sv >= 0) {
        const int p = pos + __popc(m & ((1u << lane) - 1u));
        fr[p] = e * C + sv;
        fw[p] = sw[e * ld + j];
        ftok[p] = (uint8_t)j;
      }
      pos += __popc(m);
    }
  }
  __syncthreads();
  // the slots and scores were written by the routing kernels, which the
  // caller's stream joined (fully) before the chain this kernel ends began;
  // the rows z are the output of its immediate predecessor
  griddep_wait();
  // 4. stream the rows
  const int n_total = start[tpc];
  const int n_tok = min(tpc, T - t0);
  const int d8 = d >> 3;
  for (int q = threadIdx.x; q < d8; q += kCombThreads) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    int cur = 0;  // token whose sum is being accumulated
    for (int p0 = 0; p0 < n_total; p0 += kCombBatch) {
      uint4 v[kCombBatch];
#pragma unroll
      for (int u = 0; u < kCombBatch; ++u)
        if (p0 + u < n_total)
          v[u] = __ldcs(reinterpret_cast<const uint4*>(z + (int64_t)fr[p0 + u] * d) + q);
#pragma unroll
      for (int u = 0; u < kCombBatch; ++u) {
        if (p0 + u < n_total) {
          const int tok = ftok[p0 + u];
          while (cur < tok) {  // close the tokens before this pick
            reinterpret_cast<uint4*>(y + (int64_t)(t0 + cur) * d)[q] = f32x8_to_bf16x8(acc);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
            ++cur;
          }
          float f[8];
          bf16x8_to_f32(v[u], f);
          const float w = fw[p0 + u];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(w, f[i]));
        }
      }
    }
    while (cur < n_tok) {
      reinterpret_cast<uint4*>(y + (int64_t)(t0 + cur) * d)[q] = f32x8_to_bf16x8(acc);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      ++cur;
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

// The cross-CTA counter wait of the requantising GEMM, alone: thread 0
// clears the counter and the abort word at `words` (two ints), then waits for
// the counter to reach 1, which nothing does; *result = 0 once it gave up.
__global__ void count_wait_selftest_kernel(unsigned long long limit_ns, int* words, int* result) {
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    words[0] = 0;
    words[1] = 0;
    __threadfence();
    const bool ok = wait_count_geq(words, 1, words + 1, &abort_flag, kErrSelfTest, limit_ns);
    *result = ok ? 1 : 0;
  }
}

}  // namespace convrot
