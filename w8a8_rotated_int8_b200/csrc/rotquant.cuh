// Fused block-Hadamard rotation + per-row symmetric INT8 quantisation.
//
// "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder", section
// "Quantization": each row is rotated in contiguous groups of g along K
// (ConvRot) and quantised to symmetric INT8 with nearest rounding and one
// FP32 scale per row. "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section
// "How they were made": block Hadamard rotation, one scale per row, 8-bit
// activations, with the rotation and rounding done in fp32. The same
// operation serves the weights (offline, per output row), the activations
// (per token) and the SwiGLU output before the down projection.
//
// Arithmetic (fp32, IEEE, no contraction):
//   rotation  fast Walsh-Hadamard butterflies (a + b, a - b) with spans
//             1, 2, ..., g/2 in that order, then v' = v * (1/sqrt(g)) (a
//             power of two for g a power of four);
//   scale     a = max|v'|, s = a / 127, r = 127 / a (one IEEE division each);
//   codes     q = rint(v' * r), ties to even (|v' * r| <= 127 (1 + 2^-24), so
//             the code never leaves [-127, 127]);
//   a row with a < 2^-120 gets s = 0 and all-zero codes.
//
// Layout: each thread owns 16 consecutive elements of a row (one 32-byte bf16
// or 64-byte fp32 load, one 16-byte code store). Spans 1..8 are butterflies
// in registers; the larger spans pair 16-element chunks held by lanes whose
// indices differ in one bit, exchanged with warp shuffles (a row's chunks sit
// in consecutive lanes, so chunk i and chunk i ^ d are lane and lane ^ d).
#pragma once

#include "common.cuh"

namespace convrot {

constexpr int kRqThreads = 256;

template <typename InT>
__device__ __forceinline__ void rq_load16(const InT* p, float (&v)[16]);

template <>
__device__ __forceinline__ void rq_load16<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  const uint4 a = __ldg(q);
  const uint4 b = __ldg(q + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void rq_load16<float>(const float* p, float (&v)[16]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 f = __ldg(q + k);
    v[4 * k] = f.x;
    v[4 * k + 1] = f.y;
    v[4 * k + 2] = f.z;
    v[4 * k + 3] = f.w;
  }
}

template <int G>
struct RqTraits {
  static_assert(G == 1 || G == 4 || G == 16 || G == 64 || G == 256, "group must be a power of four <= 256");
  static constexpr int kInRegSpanEnd = G < 16 ? G : 16;  // spans 1 .. kInRegSpanEnd/2 in registers
  static constexpr int kLaneSpanEnd = G >= 16 ? G / 16 : 1;  // lane distances 1 .. kLaneSpanEnd/2
  static constexpr float kInvSqrt = G == 1 ? 1.0f : G == 4 ? 0.5f : G == 16 ? 0.25f : G == 64 ? 0.125f : 0.0625f;
};

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// Row-wise max over the `tpr` threads of a row. tpr is a power of two <= 32
// (rows live in aligned lane segments) or a multiple of 32.
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
template <typename InT, int G>
__global__ void __launch_bounds__(512) rotquant_kernel(const InT* __restrict__ x, int64_t rows,
                                                      int K, int tpr, int8_t* __restrict__ q,
                                                      float* __restrict__ scales, RqOut out) {
  using Tr = RqTraits<G>;
  __shared__ float red[16];  // per-warp maxima (512 threads at most)
  const int lane = threadIdx.x & 31;
  const int rows_per_cta = blockDim.x / tpr;
  const int r_local = threadIdx.x / tpr;
  const int i = threadIdx.x - r_local * tpr;  // 16-chunk index in the row
  const int64_t row = (int64_t)blockIdx.x * rows_per_cta + r_local;
  const int nchunks = K >> 4;
  const bool active = (row < rows) && (i < nchunks);

  float v[16];
  if (active) {
    rq_load16<InT>(x + row * K + (int64_t)i * 16, v);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = 0.0f;
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
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    v[j] = __fmul_rn(v[j], Tr::kInvSqrt);
    m = fmaxf(m, fabsf(v[j]));
  }
  m = rq_row_max(m, tpr, red);

  const bool nonzero = m >= 7.52316384526264e-37f;  // 2^-120
  const float s = nonzero ? __fdiv_rn(m, 127.0f) : 0.0f;
  const float r = nonzero ? __fdiv_rn(127.0f, m) : 0.0f;
  if (active) {
    // rint by adding 1.5 * 2^23 (the fp32 add rounds to nearest even)
    int k[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      k[j] = __float_as_int(__fadd_rn(__fmul_rn(v[j], r), 12582912.0f)) - 0x4B400000;
    uint4 c;
    c.x = pack4(k[0], k[1], k[2], k[3]);
    c.y = pack4(k[4], k[5], k[6], k[7]);
    c.z = pack4(k[8], k[9], k[10], k[11]);
    c.w = pack4(k[12], k[13], k[14], k[15]);
    *reinterpret_cast<uint4*>(q + rq_dst(out, row, K, i * 16)) = c;
    if (i == 0) scales[row] = s;
  }
}

}  // namespace convrot
