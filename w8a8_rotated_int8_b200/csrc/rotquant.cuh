// Fused block-Hadamard rotation + per-row symmetric INT8 quantisation.
//
// "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder", section
// "Quantization": each row is rotated in contiguous groups of g along K
// (ConvRot) and quantised to symmetric INT8 with nearest rounding and one
// FP32 scale per row. "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section
// "How they were made": block Hadamard rotation, one scale per row, 8-bit
// activations. The definition (Sylvester Hadamard, natural order):
//   v' = v . blockdiag(H_g / sqrt(g)),  a = max|v'|,
//   s  = fp32(a / 127),  q = clamp(rne(v' / s), -127, 127)  (s = 0: q = 0).
//
// Two implementations:
//  * rotquant_f64_kernel (offline weights): the rotation and the quotient in
//    fp64, which reproduces the definition exactly: the butterflies of bf16
//    values are exact sums (while a group's exponent spread stays under ~37
//    bits), the scale is the fp64 quotient rounded once to fp32, and every
//    code is rne of a correctly rounded fp64 quotient.
//  * rotquant_kernel / rotquant_tma_kernel (activations and h, on the hot
//    path): fp32 arithmetic, IEEE, no contraction --
//      rotation  butterflies (a + b, a - b), spans 1, 2, ..., g/2, giving
//                u = v' * sqrt(g); v' = u * (1/sqrt(g)) (a power of two for g
//                a power of four, so the scaling is exact and commutes with
//                fp32 rounding);
//      scale     a = max|v'| = max|u| / sqrt(g), s = a / 127 (one IEEE
//                division; subnormal or 0 for tiny a);
//      codes     while a >= 2^-100: q = rne(u * (127 / max|u|)), the product
//                exact inside one fma with the rounding constant 1.5 * 2^23
//                (|u r| <= 127 (1 + 2^-24): the code never leaves
//                [-127, 127]); below that q = clamp(rint(v' / s)) through an
//                exactly rescaled reciprocal, so a subnormal s is honoured;
//                s = 0 gives all-zero codes.
//    These codes differ from the definition's only where v'/s lies within
//    the fp32 rounding error of a half-integer (a flip of one, at most).
//
// Layout of the fp32 forms: each thread owns 16 consecutive elements of a
// row (one 32-byte bf16 or 64-byte fp32 load, one 16-byte code store). Spans
// 1..8 are butterflies in registers; the larger spans pair 16-element chunks
// held by lanes whose indices differ in one bit, exchanged with warp shuffles
// (a row's chunks sit in consecutive lanes, so chunk i and chunk i ^ d are
// lane and lane ^ d).
#pragma once

#include "common.cuh"

namespace convrot {

constexpr int kRqThreads = 256;

// The raw 16 elements of one thread's chunk, as loaded (2 x 16 bytes of bf16
// or 4 x 16 bytes of fp32), so the next row's load can be in flight while
// this row is computed.
template <typename InT>
struct RqRaw {
  static constexpr int kVecs = (int)(16 * sizeof(InT) / 16);
  uint4 u[kVecs];
};

template <typename InT>
__device__ __forceinline__ void rq_load_raw(const InT* p, RqRaw<InT>& r) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int k = 0; k < RqRaw<InT>::kVecs; ++k) r.u[k] = __ldg(q + k);
}

__device__ __forceinline__ void rq_unpack(const RqRaw<__nv_bfloat16>& r, float (&v)[16]) {
  const uint32_t w[8] = {r.u[0].x, r.u[0].y, r.u[0].z, r.u[0].w,
                         r.u[1].x, r.u[1].y, r.u[1].z, r.u[1].w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void rq_unpack(const RqRaw<float>& r, float (&v)[16]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[4 * k] = __uint_as_float(r.u[k].x);
    v[4 * k + 1] = __uint_as_float(r.u[k].y);
    v[4 * k + 2] = __uint_as_float(r.u[k].z);
    v[4 * k + 3] = __uint_as_float(r.u[k].w);
  }
}

template <int G>
struct RqTraits {
  static_assert(G == 1 || G == 4 || G == 16 || G == 64 || G == 256, "group must be a power of four <= 256");
  static constexpr int kInRegSpanEnd = G < 16 ? G : 16;  // spans 1 .. kInRegSpanEnd/2 in registers
  static constexpr int kLaneSpanEnd = G >= 16 ? G / 16 : 1;  // lane distances 1 .. kLaneSpanEnd/2
  static constexpr float kInvSqrt = G == 1 ? 1.0f : G == 4 ? 0.5f : G == 16 ? 0.25f : G == 64 ? 0.125f : 0.0625f;
};

// Rows whose absmax a is at least this use the reciprocal r = 127 / a (finite
// and normal); the codes of smaller rows come from their (possibly subnormal)
// scale s: q = clamp(rint((v * 2^100) * r2)), r2 = 1 / (s * 2^100), where both
// products by 2^100 are exact and s * 2^100 is a normal number.
constexpr float kRqRecipMin = 7.888609052210118e-31f;  // 2^-100
constexpr float kRqTinyLift = 1.2676506002282294e+30f;  // 2^100

// r2 of a tiny row (0 when s is 0: every code is then 0).
__device__ __forceinline__ float rq_tiny_recip(float s) {
  return s == 0.0f ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(s, kRqTinyLift));
}

__device__ __forceinline__ int rq_code_tiny(float v, float r2) {
  const int c = __float2int_rn(__fmul_rn(__fmul_rn(v, kRqTinyLift), r2));
  return c > 127 ? 127 : (c < -127 ? -127 : c);
}

// Bits whose low byte is the code rne(u * r) (|u r| <= 127.5): the exact
// product plus 1.5 * 2^23, rounded once (one fma), lands in [2^23, 2^24)
// where fp32 has unit spacing, so the rounding is to the nearest integer,
// ties to even.
constexpr float kRqMagic = 12582912.0f;  // 1.5 * 2^23
__device__ __forceinline__ uint32_t rq_code_bits(float u, float r) {
  return __float_as_uint(__fmaf_rn(u, r, kRqMagic));
}

// Two codes at once from a packed pair (fma.rn.f32x2): the bits of both.
__device__ __forceinline__ unsigned long long rq_code_bits2(unsigned long long u2,
                                                            unsigned long long r2,
                                                            unsigned long long magic2) {
  return f2_fma(u2, r2, magic2);
}

// Low bytes of four code bit patterns (c0 lowest) as one word.
__device__ __forceinline__ uint32_t rq_pack_bytes(uint32_t c0, uint32_t c1, uint32_t c2,
                                                  uint32_t c3) {
  return __byte_perm(__byte_perm(c0, c1, 0x0040), __byte_perm(c2, c3, 0x0040), 0x5410);
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// Row-wise max over the `tpr` threads of a row. tpr is a power of two <= 32
// (rows live in aligned lane segments) or a multiple of 32 (then every thread
// of the CTA must call it: it synchronises the CTA once).
__device__ __forceinline__ float rq_row_max(float m, int tpr, float* red) {
  const int lane = threadIdx.x & 31;
  if (tpr <= 32) {
    for (int off = tpr >> 1; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    return m;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const int warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = m;
  __syncthreads();
  const int wpr = tpr >> 5;
  const int w0 = (threadIdx.x / tpr) * wpr;
  float r = 0.0f;
  for (int w = 0; w < wpr; ++w) r = fmaxf(r, red[w0 + w]);
  return r;
}

// Where the codes of a row go. Row-major: q[row * K + k]. Tiled (the
// weight format of the grouped GEMM): the rows are split into matrices of
// `mat_rows` rows; each matrix into 128-row blocks, each block into 128-byte
// K tiles; tile (block rb, k-tile kb) is 16 KB at ((rb * kb_count + kb) *
// 16384) holding 128 rows of 128 bytes. rb = mat * rb_per_mat + row_in_mat/128.
struct RqOut {
  int tiled;
  int64_t mat_rows;
  int rb_per_mat;
  int kb_count;
};

__device__ __forceinline__ int64_t rq_dst(const RqOut& o, int64_t row, int K, int k0) {
  if (!o.tiled) return row * K + k0;
  const int64_t mat = row / o.mat_rows;
  const int64_t r = row - mat * o.mat_rows;
  const int64_t rb = mat * o.rb_per_mat + (r >> 7);
  return ((rb * o.kb_count + (k0 >> 7)) * 128 + (r & 127)) * 128 + (k0 & 127);
}

// x: [rows, K] (bf16 or fp32), q: codes (layout `out`), scales: [rows] fp32.
// blockDim.x = rows_per_cta * tpr exactly (rows_per_cta = max(1, 256 / tpr)).
// Persistent: CTA b handles the row groups b, b + gridDim.x, ... (a group is
// rows_per_cta consecutive rows) and loads its next group's chunk before
// computing the current one.
template <typename InT, int G>
__global__ void __launch_bounds__(1024) rotquant_kernel(const InT* __restrict__ x, int64_t rows,
                                                      int K, int tpr, int8_t* __restrict__ q,
                                                      float* __restrict__ scales, RqOut out) {
  griddep_launch_dependents();
  griddep_wait();
  using Tr = RqTraits<G>;
  __shared__ float red[2][32];  // per-warp maxima (1024 threads at most), by iteration parity
  const int lane = threadIdx.x & 31;
  const int rows_per_cta = blockDim.x / tpr;
  const int r_local = threadIdx.x / tpr;
  const int i = threadIdx.x - r_local * tpr;  // 16-chunk index in the row
  const int nchunks = K >> 4;
  const int64_t groups = (rows + rows_per_cta - 1) / rows_per_cta;

  RqRaw<InT> raw;
  int64_t grp = blockIdx.x;
  {
    const int64_t row = grp * rows_per_cta + r_local;
    if (grp < groups && row < rows && i < nchunks) rq_load_raw<InT>(x + row * K + (int64_t)i * 16, raw);
  }
  for (int it = 0; grp < groups; grp += gridDim.x, ++it) {
    const int64_t row = grp * rows_per_cta + r_local;
    const bool active = (row < rows) && (i < nchunks);
    float v[16];
    if (active) {
      rq_unpack(raw, v);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = 0.0f;
    }
    {
      const int64_t row_n = (grp + gridDim.x) * rows_per_cta + r_local;
      if (grp + gridDim.x < groups && row_n < rows && i < nchunks)
        rq_load_raw<InT>(x + row_n * K + (int64_t)i * 16, raw);
    }
    // spans 1, 2, 4, 8 inside the thread's 16 elements
#pragma unroll
    for (int span = 1; span < Tr::kInRegSpanEnd; span <<= 1) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if ((j & span) == 0) {
          const float a = v[j];
          const float b = v[j + span];
          v[j] = __fadd_rn(a, b);
          v[j + span] = __fsub_rn(a, b);
        }
      }
    }
    // spans 16, 32, ... between chunks: the lower chunk of a pair keeps a + b,
    // the upper one a - b, as one rounding each: fma(+-1, own, partner)
#pragma unroll
    for (int d = 1; d < Tr::kLaneSpanEnd; d <<= 1) {
      const float sgn = (lane & d) ? -1.0f : 1.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float p = __shfl_xor_sync(0xffffffffu, v[j], d);
        v[j] = __fmaf_rn(sgn, v[j], p);
      }
    }
    float mu = 0.0f;  // max |u| (unscaled)
#pragma unroll
    for (int j = 0; j < 16; ++j) mu = fmaxf(mu, fabsf(v[j]));
    mu = rq_row_max(mu, tpr, red[it & 1]);

    const float m = __fmul_rn(mu, Tr::kInvSqrt);
    const float s = __fdiv_rn(m, 127.0f);
    const bool recip = m >= kRqRecipMin;
    const float r = recip ? __fdiv_rn(127.0f, mu) : 0.0f;
    if (active) {
      int k[16];
      if (recip) {
#pragma unroll
        for (int j = 0; j < 16; ++j) k[j] = (int)rq_code_bits(v[j], r) - 0x4B400000;
      } else {
        const float r2 = rq_tiny_recip(s);
#pragma unroll
        for (int j = 0; j < 16; ++j) k[j] = rq_code_tiny(__fmul_rn(v[j], Tr::kInvSqrt), r2);
      }
      uint4 c;
      c.x = pack4(k[0], k[1], k[2], k[3]);
      c.y = pack4(k[4], k[5], k[6], k[7]);
      c.z = pack4(k[8], k[9], k[10], k[11]);
      c.w = pack4(k[12], k[13], k[14], k[15]);
      *reinterpret_cast<uint4*>(q + rq_dst(out, row, K, i * 16)) = c;
      if (i == 0) scales[row] = s;
    }
  }
}

// ------------------------------------------------------- warp-per-row form --
// The same operation for K % 64 == 0 and K <= 2048, with fewer instructions
// per element: lane l of a row segment (SEG lanes, a power of two) owns the 64
// consecutive elements [64 l, 64 l + 64) of the row, held as 32 pairs
// p[m] = (v[2m], v[2m+1]). Span 1 pairs the two halves of each register
// (scalar ops); spans 2 .. 32 pair whole registers and use the packed
// add/sub.rn.f32x2 (two IEEE fp32 operations each); for G = 256 the spans 64
// and 128 pair lanes l ^ 1 and l ^ 2 (warp shuffles, one packed fma each).
// The row maximum is a shuffle reduction over the segment. SEG * 64 >= K; a
// warp holds 32 / SEG rows. The rows reach shared memory by TMA (below).
// 16 bytes of a lane's 64 elements (piece j: elements 8j.. of bf16, 4j.. of
// fp32) into their pairs of p.
template <typename InT>
__device__ __forceinline__ void rq_unpack_piece(const uint4 v, int j, unsigned long long (&p)[32]);

template <>
__device__ __forceinline__ void rq_unpack_piece<__nv_bfloat16>(const uint4 v, int j,
                                                               unsigned long long (&p)[32]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    p[4 * j + i] = f2_pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

template <>
__device__ __forceinline__ void rq_unpack_piece<float>(const uint4 v, int j,
                                                       unsigned long long (&p)[32]) {
  p[2 * j] = f2_pack(__uint_as_float(v.x), __uint_as_float(v.y));
  p[2 * j + 1] = f2_pack(__uint_as_float(v.z), __uint_as_float(v.w));
}

// Rotation, scale and codes of the 64 elements (32 pairs) a lane holds;
// every lane of the warp calls it (shuffles).
template <int G, int SEG>
__device__ __forceinline__ void rq_lane64(unsigned long long (&p)[32], bool active, int li,
                                          int64_t row, int K, int8_t* __restrict__ q,
                                          float* __restrict__ scales, const RqOut& out) {
  using Tr = RqTraits<G>;
  // span 1: the two halves of each pair
  if (G >= 2) {
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      const float2 ab = f2_unpack(p[m]);
      p[m] = f2_pack(__fadd_rn(ab.x, ab.y), __fsub_rn(ab.x, ab.y));
    }
  }
  // spans 2 .. min(G, 64) / 2: pairs of registers m, m + span / 2
#pragma unroll
  for (int hs = 1; 2 * hs < (G < 64 ? G : 64); hs <<= 1) {
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      if ((m & hs) == 0) {
        const unsigned long long a = p[m], b = p[m + hs];
        p[m] = f2_add(a, b);
        p[m + hs] = f2_sub(a, b);
      }
    }
  }
  // spans 64, 128 (G = 256): lanes l ^ 1, l ^ 2 of the segment
  if (G == 256) {
#pragma unroll
    for (int d = 1; d <= 2; d <<= 1) {
      const float sg = (li & d) ? -1.0f : 1.0f;
      const unsigned long long sg2 = f2_pack(sg, sg);
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        const float2 own = f2_unpack(p[m]);
        const float px = __shfl_xor_sync(0xffffffffu, own.x, d);
        const float py = __shfl_xor_sync(0xffffffffu, own.y, d);
        p[m] = f2_fma(sg2, p[m], f2_pack(px, py));
      }
    }
  }
  // max |u| of the unscaled butterfly outputs (v' = u / sqrt(g) is never formed)
  float mu = 0.0f;
#pragma unroll
  for (int m = 0; m < 32; ++m) {
    const float2 t = f2_unpack(p[m]);
    mu = fmaxf(mu, fmaxf(fabsf(t.x), fabsf(t.y)));
  }
#pragma unroll
  for (int off = SEG >> 1; off > 0; off >>= 1)
    mu = fmaxf(mu, __shfl_xor_sync(0xffffffffu, mu, off));
  const float mx = __fmul_rn(mu, Tr::kInvSqrt);
  const float sc = __fdiv_rn(mx, 127.0f);
  const bool recip = mx >= kRqRecipMin;
  const float r = recip ? __fdiv_rn(127.0f, mu) : 0.0f;
  if (active) {
    uint32_t cw[16];
    if (recip) {
      const unsigned long long r2 = f2_pack(r, r);
      const unsigned long long magic2 = f2_pack(kRqMagic, kRqMagic);
#pragma unroll
      for (int m = 0; m < 32; m += 2) {
        const float2 a = f2_unpack(rq_code_bits2(p[m], r2, magic2));
        const float2 b = f2_unpack(rq_code_bits2(p[m + 1], r2, magic2));
        cw[m >> 1] = rq_pack_bytes(__float_as_uint(a.x), __float_as_uint(a.y),
                                   __float_as_uint(b.x), __float_as_uint(b.y));
      }
    } else {
      const float r2 = rq_tiny_recip(sc);
#pragma unroll
      for (int m = 0; m < 32; m += 2) {
        const float2 a = f2_unpack(p[m]);
        const float2 b = f2_unpack(p[m + 1]);
        cw[m >> 1] = pack4(rq_code_tiny(__fmul_rn(a.x, Tr::kInvSqrt), r2),
                           rq_code_tiny(__fmul_rn(a.y, Tr::kInvSqrt), r2),
                           rq_code_tiny(__fmul_rn(b.x, Tr::kInvSqrt), r2),
                           rq_code_tiny(__fmul_rn(b.y, Tr::kInvSqrt), r2));
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4*>(q + rq_dst(out, row, K, li * 64 + 16 * c)) =
          make_uint4(cw[4 * c], cw[4 * c + 1], cw[4 * c + 2], cw[4 * c + 3]);
    if (li == 0) scales[row] = sc;
  }
}

// TMA-fed form: every warp keeps a ring of kRqSlots shared-memory slots, each
// holding one unit (32 / SEG rows) as loaded by a 3-D tiled TMA copy
// {128 bytes, K * sizeof(InT) / 128 chunks, rows} with the 128-byte swizzle;
// lane 0 refills a slot as soon as the warp has read it, so kRqSlots - 1
// units stream in while one is computed. A lane reads its 16-byte pieces k at
// position k ^ (smem row & 7): the swizzle makes those reads conflict-free
// for the 8 lanes of each phase while the piece index stays static.
constexpr int kRqTmaWarps = 8;
constexpr int kRqMaxSlots = 4;  // ring depth per warp

// wait_at_end: the kernel reads nothing its predecessor on the stream writes
// (it runs beside it) and waits for that predecessor only before it exits, so
// that its completion implies the predecessor's (the MoE call's schedule);
// otherwise it waits for the predecessor before reading anything.
template <typename InT, int G, int SEG>
__global__ void __launch_bounds__(kRqTmaWarps * 32, 2) rotquant_tma_kernel(
    const __grid_constant__ CUtensorMap tm, int64_t rows, int K, int slots, int slot_bytes,
    int8_t* __restrict__ q, float* __restrict__ scales, RqOut out, int wait_at_end) {
  griddep_launch_dependents();
  if (!wait_at_end) griddep_wait();
  static_assert(SEG >= 1 && SEG <= 32 && (SEG & (SEG - 1)) == 0, "segment of 2^k lanes");
  static_assert(G != 256 || SEG >= 4, "a 256-group spans four lanes");
  constexpr int kRowsPerWarp = 32 / SEG;
  constexpr int kChunksPerLane = (int)(64 * sizeof(InT) / 128);  // 128-byte smem rows
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int li = lane & (SEG - 1);
  uint8_t* ring = smem + (size_t)warp * slots * slot_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kRqTmaWarps * slots * slot_bytes) +
                   warp * slots;
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + (size_t)kRqTmaWarps * slots * (slot_bytes + 8)) +
      warp;
  const int kb = K * (int)sizeof(InT) / 128;
  const uint32_t tx_bytes = (uint32_t)(kRowsPerWarp * kb * 128);
  const int64_t units = (rows + kRowsPerWarp - 1) / kRowsPerWarp;
  const int64_t u0 = (int64_t)blockIdx.x * kRqTmaWarps + warp;
  const int64_t nw = (int64_t)gridDim.x * kRqTmaWarps;
  const bool lane_on = li * 64 < K;
  const uint64_t policy = l2_policy_evict_first();

  if (lane == 0) {
    for (int k = 0; k < slots; ++k) mbar_init(&bars[k], 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm);
    for (int k = 0; k < slots; ++k) {
      const int64_t u = u0 + k * nw;
      if (u >= units) break;
      mbar_arrive_expect_tx(&bars[k], tx_bytes);
      tma_load_3d(ring + (size_t)k * slot_bytes, &tm, &bars[k], 0, 0, (int)(u * kRowsPerWarp),
                  policy);
    }
  }
  __syncwarp();
  // iteration `it` consumes unit u0 + it * nw from slot it % slots (phase
  // parity (it / slots) & 1); its load was issued `slots` iterations earlier
  int64_t it = 0;
  for (int64_t u = u0; u < units; u += nw, ++it) {
    const int k = (int)(it % slots);
    const uint32_t parity = (uint32_t)((it / slots) & 1);
    const bool ok = mbar_wait(&bars[k], parity, abort_flag, kErrTimeoutStream);
    if (__any_sync(0xffffffffu, !ok)) {  // the whole warp leaves together
      *abort_flag = 1;
      break;
    }

    const int64_t row = u * kRowsPerWarp + lane / SEG;
    const bool active = row < rows && lane_on;
    unsigned long long p[32];
    if (active) {
      const int srow0 = (lane / SEG) * kb + li * kChunksPerLane;
#pragma unroll
      for (int h = 0; h < kChunksPerLane; ++h) {
        const int srow = srow0 + h;
        const uint8_t* base = ring + (size_t)k * slot_bytes + (size_t)srow * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          rq_unpack_piece<InT>(*reinterpret_cast<const uint4*>(base + ((c ^ (srow & 7)) << 4)),
                               h * 8 + c, p);
      }
    } else {
#pragma unroll
      for (int m = 0; m < 32; ++m) p[m] = 0ull;
    }
    __syncwarp();
    // the generic-proxy reads of this slot are ordered before the next TMA write
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (lane == 0) {
      const int64_t un = u + (int64_t)slots * nw;
      if (un < units) {
        mbar_arrive_expect_tx(&bars[k], tx_bytes);
        tma_load_3d(ring + (size_t)k * slot_bytes, &tm, &bars[k], 0, 0, (int)(un * kRowsPerWarp),
                    policy);
      }
    }

    rq_lane64<G, SEG>(p, active, li, row, K, q, scales, out);
  }
  if (*abort_flag) {
    // a wait ran out: let every copy this warp still has in flight land
    // (bounded) before the CTA's shared memory is released
    // (the loads of iterations it .. it + slots - 1 were issued, not consumed)
    if (lane == 0) {
      for (int j = 0; j < slots; ++j) {
        const int64_t itj = it + j;
        if (u0 + itj * nw < units)
          mbar_drain(&bars[itj % slots], (uint32_t)((itj / slots) & 1), g_wait_limit_ns);
      }
    }
    __syncwarp();
  }
  if (wait_at_end) griddep_wait();
}

// ------------------------------------------------------ fp64 (offline) --
// The definition exactly, for bf16 weight rows (see the top of this file):
// one CTA per row at a time (persistent over rows b, b + gridDim.x, ...), the
// row held in shared memory as fp64, butterflies stage by stage over the
// whole row (spans 1 .. G/2 stay inside each contiguous group of G), the
// exact scaling by 1/sqrt(G), a block maximum, s = fp32(a / 127) from the
// correctly rounded fp64 quotient, codes rne(v' / s) from correctly rounded
// fp64 quotients, clamped to [-127, 127]. K % 16 == 0; dynamic shared memory
// K * 8 bytes.
constexpr int kRq64Threads = 256;

template <int G>
__global__ void __launch_bounds__(kRq64Threads) rotquant_f64_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t rows, int K, int8_t* __restrict__ q,
    float* __restrict__ scales, RqOut out) {
  extern __shared__ double row_s[];
  __shared__ double red[kRq64Threads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double inv = (double)RqTraits<G>::kInvSqrt;  // 1/sqrt(G), a power of two
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x + row * K);
    for (int i = tid; i < K / 8; i += kRq64Threads) {
      const uint4 u = __ldg(src + i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        row_s[8 * i + 2 * k] = (double)__uint_as_float(w[k] << 16);
        row_s[8 * i + 2 * k + 1] = (double)__uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
    __syncthreads();
#pragma unroll 1
    for (int span = 1; span < G; span <<= 1) {
      for (int p = tid; p < K / 2; p += kRq64Threads) {
        const int i = ((p & ~(span - 1)) << 1) | (p & (span - 1));
        const double a = row_s[i], b = row_s[i + span];
        row_s[i] = __dadd_rn(a, b);
        row_s[i + span] = __dsub_rn(a, b);
      }
      __syncthreads();
    }
    double m = 0.0;
    for (int i = tid; i < K; i += kRq64Threads) {
      const double v = __dmul_rn(row_s[i], inv);
      row_s[i] = v;
      m = fmax(m, fabs(v));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = 0.0;
#pragma unroll
    for (int w = 0; w < kRq64Threads / 32; ++w) m = fmax(m, red[w]);
    const float s = __double2float_rn(__ddiv_rn(m, 127.0));
    const double sd = (double)s;
    for (int c = tid; c < K / 16; c += kRq64Threads) {
      int k[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        int code = 0;
        if (s != 0.0f) {
          code = __double2int_rn(__ddiv_rn(row_s[16 * c + j], sd));
          code = code > 127 ? 127 : (code < -127 ? -127 : code);
        }
        k[j] = code;
      }
      uint4 cv;
      cv.x = pack4(k[0], k[1], k[2], k[3]);
      cv.y = pack4(k[4], k[5], k[6], k[7]);
      cv.z = pack4(k[8], k[9], k[10], k[11]);
      cv.w = pack4(k[12], k[13], k[14], k[15]);
      *reinterpret_cast<uint4*>(q + rq_dst(out, row, K, 16 * c)) = cv;
    }
    if (tid == 0) scales[row] = s;
    __syncthreads();  // the row buffer and red[] are reused by the next row
  }
}

}  // namespace convrot
