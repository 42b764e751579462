// Fused block-Hadamard rotation + per-row symmetric INT8 quantisation.
//
// "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder", section
// "Quantization": each row is rotated in contiguous groups of g along K
// (ConvRot) and quantised to symmetric INT8 with nearest rounding and one
// FP32 scale per row. "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section
// "How they were made": block Hadamard rotation, one scale per row, 8-bit
// activations. The same operation serves the weights (offline, per output
// row), the activations (per token) and the SwiGLU output before the down
// projection.
//
// Arithmetic: the rotation runs in fp64 butterflies. Inputs are bf16 or fp32
// and g is a power of four, so every partial sum and the 1/sqrt(g) scaling
// are exact for ordinary data and the rotated value equals the exact one.
// Scale s = fp32(absmax / 127); code q = clamp(rint(v / s), -127, 127), ties
// to even. The division is replaced by a multiply with the reciprocal plus a
// distance check: only values that land within 1e-9 of a rounding boundary
// take the true fp64 division, so the codes equal those of the definition.
//
// Layout: each thread owns 16 consecutive elements of a row (one 32-byte bf16
// or 64-byte fp32 load, one 16-byte code store). Groups up to 16 are finished
// in registers; for g = 64 / 256 the remaining butterfly stages run after one
// transpose of the row through shared memory (XOR-swizzled, free of bank
// conflicts for both group sizes), then the codes go back through shared memory so the global
// store stays contiguous.
#pragma once

#include "common.cuh"

namespace convrot {

constexpr int kRqThreads = 256;

template <typename InT>
__device__ __forceinline__ void rq_load16(const InT* p, double (&v)[16]);

template <>
__device__ __forceinline__ void rq_load16<__nv_bfloat16>(const __nv_bfloat16* p, double (&v)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  const uint4 a = __ldg(q);
  const uint4 b = __ldg(q + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[2 * k] = (double)__uint_as_float(w[k] << 16);
    v[2 * k + 1] = (double)__uint_as_float(w[k] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void rq_load16<float>(const float* p, double (&v)[16]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 f = __ldg(q + k);
    v[4 * k] = (double)f.x;
    v[4 * k + 1] = (double)f.y;
    v[4 * k + 2] = (double)f.z;
    v[4 * k + 3] = (double)f.w;
  }
}

// Butterflies (a+b, a-b) for spans 1 .. 2^(STAGES-1) over N consecutive values.
template <int STAGES, int N>
__device__ __forceinline__ void fwht_inreg(double* v) {
#pragma unroll
  for (int s = 0; s < STAGES; ++s) {
    const int span = 1 << s;
#pragma unroll
    for (int j = 0; j < N; ++j) {
      if ((j & span) == 0) {
        const double a = v[j];
        const double b = v[j + span];
        v[j] = __dadd_rn(a, b);
        v[j + span] = __dsub_rn(a, b);
      }
    }
  }
}

template <int G>
struct RqTraits {
  static_assert(G == 1 || G == 4 || G == 16 || G == 64 || G == 256, "group must be a power of four <= 256");
  static constexpr int kLog2 = G == 1 ? 0 : G == 4 ? 2 : G == 16 ? 4 : G == 64 ? 6 : 8;
  static constexpr int kInReg = kLog2 < 4 ? kLog2 : 4;       // stages inside a 16-chunk
  static constexpr int kChunks = G >= 16 ? G / 16 : 1;       // 16-chunks per group
  static constexpr int kCross = kLog2 - kInReg;              // stages across chunks
  static constexpr double kInvSqrt = G == 1 ? 1.0 : G == 4 ? 0.5 : G == 16 ? 0.25 : G == 64 ? 0.125 : 0.0625;
};

// One code from an unnormalised rotated value u (v' = u * inv_sqrt exactly).
__device__ __forceinline__ int rq_code(double u, double r_scaled, double inv_sqrt, double s64) {
  const double magic = 6755399441055744.0;  // 1.5 * 2^52: adding it rounds to an integer
  const double y = __dmul_rn(u, r_scaled);  // v' / s up to a few fp64 ulps
  const double t = __dadd_rn(y, magic);
  const double ry = __dsub_rn(t, magic);     // rint(y), ties to even
  int k;
  if (fabs(__dsub_rn(y, ry)) < 0.4999999990) {
    k = __double2loint(t);                   // two's complement integer in the low word
  } else {
    k = __double2int_rn(__ddiv_rn(__dmul_rn(u, inv_sqrt), s64));
  }
  return max(-127, min(127, k));
}

// Position of (16-chunk ci, column c) in the transpose buffer: columns are
// XOR-permuted by the chunk index with its 2-bit halves swapped, which keeps
// both the row-wise writes and the column-wise reads of g = 64 and g = 256
// free of 64-bit bank conflicts.
__device__ __forceinline__ int rq_swz(int ci, int c) {
  return ci * 16 + (c ^ (((ci & 3) << 2) | ((ci >> 2) & 3)));
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// Row-wise max over the `tpr` threads of a row. tpr is a power of two <= 32
// (rows live in aligned lane segments) or a multiple of 32.
__device__ __forceinline__ double rq_row_max(double m, int tpr, double* red) {
  const int lane = threadIdx.x & 31;
  if (tpr <= 32) {
    for (int off = tpr >> 1; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    return m;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
  const int warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = m;
  __syncthreads();
  const int wpr = tpr >> 5;
  const int w0 = (threadIdx.x / tpr) * wpr;
  double r = 0.0;
  for (int w = 0; w < wpr; ++w) r = fmax(r, red[w0 + w]);
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
  extern __shared__ __align__(16) unsigned char rq_smem[];
  double* red = reinterpret_cast<double*>(rq_smem);  // 16 warps max
  const int rows_per_cta = blockDim.x / tpr;
  const int r_local = threadIdx.x / tpr;
  const int i = threadIdx.x - r_local * tpr;  // 16-chunk index in the row
  const int64_t row = (int64_t)blockIdx.x * rows_per_cta + r_local;
  const int nchunks = K >> 4;
  const bool active = (row < rows) && (i < nchunks);

  double v[16];
  if (active) {
    rq_load16<InT>(x + row * K + (int64_t)i * 16, v);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = 0.0;
  }
  fwht_inreg<Tr::kInReg, 16>(v);

  double* buf = reinterpret_cast<double*>(rq_smem + 128) + (int64_t)r_local * K;
  unsigned char* codes =
      rq_smem + 128 + (size_t)rows_per_cta * K * sizeof(double) + (size_t)r_local * K;
  constexpr int CH = Tr::kChunks;
  constexpr int CPT = 16 / CH;  // columns held per thread after the transpose
  const int grp = i / CH;
  const int p = i - grp * CH;
  if constexpr (G >= 64) {
    if (active) {
#pragma unroll
      for (int j = 0; j < 16; ++j) buf[rq_swz(i, j)] = v[j];
    }
    __syncthreads();
    if (active) {
#pragma unroll
      for (int cc = 0; cc < CPT; ++cc) {
#pragma unroll
        for (int jj = 0; jj < CH; ++jj) {
          const int ci = grp * CH + jj;
          const int col = p * CPT + cc;
          v[cc * CH + jj] = buf[rq_swz(ci, col)];
        }
      }
    }
#pragma unroll
    for (int cc = 0; cc < CPT; ++cc) fwht_inreg<Tr::kCross, CH>(v + cc * CH);
  }

  double m = 0.0;
#pragma unroll
  for (int j = 0; j < 16; ++j) m = fmax(m, fabs(v[j]));
  m = rq_row_max(m, tpr, red);

  const double a = __dmul_rn(m, Tr::kInvSqrt);
  const float s = __double2float_rn(__ddiv_rn(a, 127.0));
  const double s64 = (double)s;
  const bool nonzero = s != 0.0f;
  const double r_scaled = nonzero ? __dmul_rn(__drcp_rn(s64), Tr::kInvSqrt) : 0.0;

  if constexpr (G >= 64) {
    if (active) {
#pragma unroll
      for (int cc = 0; cc < CPT; ++cc) {
#pragma unroll
        for (int jj = 0; jj < CH; ++jj) {
          const int ci = grp * CH + jj;
          const int col = p * CPT + cc;
          const int k = nonzero ? rq_code(v[cc * CH + jj], r_scaled, Tr::kInvSqrt, s64) : 0;
          codes[ci * 16 + col] = (unsigned char)(k & 0xFF);
        }
      }
    }
    __syncthreads();
    if (active) {
      const uint4 c = *reinterpret_cast<const uint4*>(codes + i * 16);
      *reinterpret_cast<uint4*>(q + rq_dst(out, row, K, i * 16)) = c;
    }
  } else {
    if (active) {
      int k[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) k[j] = nonzero ? rq_code(v[j], r_scaled, Tr::kInvSqrt, s64) : 0;
      uint4 c;
      c.x = pack4(k[0], k[1], k[2], k[3]);
      c.y = pack4(k[4], k[5], k[6], k[7]);
      c.z = pack4(k[8], k[9], k[10], k[11]);
      c.w = pack4(k[12], k[13], k[14], k[15]);
      *reinterpret_cast<uint4*>(q + rq_dst(out, row, K, i * 16)) = c;
    }
  }
  if (active && i == 0) scales[row] = nonzero ? s : 0.0f;
}

}  // namespace convrot
