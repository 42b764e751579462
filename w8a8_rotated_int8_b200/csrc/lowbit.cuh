// W4A8 / W6A8 in the rotated basis on the sm_100a tensor cores.
//
// Source: "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they were
// made": besides int8 ConvRot, linears come as 6-bit or 4-bit weights in the
// rotated basis with an FP8 scale for every group of 16 weights, and 8-bit
// activations. Readings (the same as the CPU definition): the int8 format's
// block Hadamard rotation; symmetric codes q in [-qmax, qmax], qmax = 7 / 31;
// FP8 = E4M3; two scale levels, an FP32 scale per row s_r = fp32(a / (qmax *
// 448)) and an E4M3 scale per group of 16, sigma = e4m3(a_group / (qmax *
// s_r)) (nearest, ties to the even code, at most 448);
// q = clamp(rne(v / (s_r * sigma))). A weight decodes to s_r * sigma * q.
//
// Weight format, for a stack of row-major matrices of `rows` x K (every
// matrix a whole number of 128-row blocks, K % 64 == 0): tiles of 128 rows x
// 64 codes, tile (row block rb, k-block kb) at (rb * K/64 + kb) * kTileBytes,
// holding b/2 planes of [128 rows][16 bytes] (plane c = bytes 16c .. 16c+15 of
// every row's packed codes), then [128 rows][4 bytes] of E4M3 group scales
// (the row's four groups in this k-block, lowest group in the lowest byte).
// A row's packed codes of one k-block store u = q + 2^(b-1):
//   32-bit words w_0 .. w_7 (bytes 4i .. 4i+3): the low four bits of u, code
//   8i+2j in bits 4j..4j+3 and code 8i+2j+1 in bits 16+4j..19+4j (j = 0..3);
//   for b = 6, words w_8 .. w_11: the top two bits, code 16i+2j in bits
//   2j..2j+1 and code 16i+2j+1 in bits 16+2j..17+2j (j = 0..7).
// A 32-bit word then yields two consecutive codes per mask, in the two
// halves of an fp16 pair.
//
// The GEMM: there is no integer tensor-core path with a scale per 16 along K,
// and INT8 activation codes are not representable in FP8, so the contraction
// runs on tcgen05 kind::f16 with fp32 accumulation over exact fp16 operands:
// an activation code (|x| <= 127) is an exact fp16, and so is q * sigma / 16
// (at most 9 significant bits, between 2^-13 and 28 * 31). The weights are
// the A operand, decoded by converter warps straight into tensor memory
// (tcgen05.st), so no decoded weight passes through shared memory; the
// activation codes are the B operand, widened to fp16 in shared memory with
// the 128-byte swizzle. D[weight row, token] = sum_k A[row, k] * B[token, k]
// accumulates sum_k q * sigma / 16 * x; the epilogue multiplies by 16
// (exact) and dequantises y = acc * (s_x * s_r).
#pragma once

#include "common.cuh"
#include "gemm_tcgen05.cuh"
#include "rotquant.cuh"

namespace convrot {

template <int BITS>
struct LbFmt {
  static_assert(BITS == 4 || BITS == 6, "4-bit or 6-bit weights");
  static constexpr int kQmax = (1 << (BITS - 1)) - 1;
  static constexpr int kBias = 1 << (BITS - 1);
  static constexpr int kPlanes = BITS / 2;
  static constexpr int kScaleOff = kPlanes * 2048;
  static constexpr int kTileBytes = kScaleOff + 512;
  // fp16 bits of -(1024 + bias): (1024 + u) * s + this * s = q * s
  static constexpr uint32_t kNegMagic2 = BITS == 4 ? 0xE408E408u : 0xE420E420u;
};

// ------------------------------------------------- offline quantiser (fp64) --
// 2^e as a double, for -1022 <= e <= 1023 (exact).
__device__ __forceinline__ double pow2_f64(int e) {
  return __longlong_as_double((long long)(1023 + e) << 52);
}

// The E4M3 code nearest to v >= 0, ties to the even code (= even mantissa),
// saturating at 448 (code 0x7E). Exact: every step is a scaling by a power
// of two or an integer rounding.
__device__ __forceinline__ uint32_t e4m3_rne(double v) {
  if (!(v < 448.0)) return 0x7Eu;
  if (v < 0.015625) return (uint32_t)__double2int_rn(v * 512.0);  // subnormals: m * 2^-9, 8 -> 0x08
  const int e = (int)((__double_as_longlong(v) >> 52) & 0x7FF) - 1023;  // v = 1.f * 2^e
  int m = __double2int_rn(v * pow2_f64(3 - e)) - 8;                    // rne(1.f * 8) - 8
  int ex = e;
  if (m == 8) {
    m = 0;
    ++ex;
  }
  const uint32_t code = ((uint32_t)(ex + 7) << 3) | (uint32_t)m;
  return code > 0x7Eu ? 0x7Eu : code;
}

// Value of a finite non-negative E4M3 code as a double (exact).
__device__ __forceinline__ double e4m3_value(uint32_t code) {
  const int e = (int)(code >> 3), m = (int)(code & 7u);
  return e == 0 ? (double)m * pow2_f64(-9) : (double)(8 + m) * pow2_f64(e - 10);
}

// One persistent CTA per row at a time: the bf16 row in shared memory as
// fp64, the butterflies stage by stage (spans 1 .. G/2 inside each group of
// G), the exact scaling by 1/sqrt(G), the row maximum, s_r from the correctly
// rounded fp64 quotient; then one thread per k-block: its four group maxima,
// the E4M3 scales of the correctly rounded quotients a_j / (qmax * s_r), the
// codes from correctly rounded quotients v / (s_r * sigma), clamped, packed.
// rows % 128 == 0, K % 64 == 0, K <= 16384; dynamic shared memory K * 8 bytes.
constexpr int kLbQuantThreads = 256;

template <int G, int BITS>
__global__ void __launch_bounds__(kLbQuantThreads) lowbit_quant_f64_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t rows, int K, uint8_t* __restrict__ out,
    float* __restrict__ row_scale) {
  using F = LbFmt<BITS>;
  extern __shared__ double row_s[];
  __shared__ double red[kLbQuantThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double inv = (double)RqTraits<G>::kInvSqrt;
  const int kbs = K / 64;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x + row * K);
    for (int i = tid; i < K / 8; i += kLbQuantThreads) {
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
      for (int p = tid; p < K / 2; p += kLbQuantThreads) {
        const int i = ((p & ~(span - 1)) << 1) | (p & (span - 1));
        const double a = row_s[i], b = row_s[i + span];
        row_s[i] = __dadd_rn(a, b);
        row_s[i + span] = __dsub_rn(a, b);
      }
      __syncthreads();
    }
    double m = 0.0;
    for (int i = tid; i < K; i += kLbQuantThreads) {
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
    for (int w = 0; w < kLbQuantThreads / 32; ++w) m = fmax(m, red[w]);
    const float s = __double2float_rn(__ddiv_rn(m, (double)F::kQmax * 448.0));
    const double qs = (double)F::kQmax * (double)s;  // exact: 5-bit times 24-bit
    const int64_t rb = row >> 7;
    const int r = (int)(row & 127);
    for (int kb = tid; kb < kbs; kb += kLbQuantThreads) {
      const double* v = row_s + kb * 64;
      uint32_t sig_word = 0;
      uint32_t lo[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      uint32_t hi[4] = {0, 0, 0, 0};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        double aj = 0.0;
#pragma unroll
        for (int i = 0; i < 16; ++i) aj = fmax(aj, fabs(v[16 * j + i]));
        const uint32_t sig = s != 0.0f ? e4m3_rne(__ddiv_rn(aj, qs)) : 0u;
        sig_word |= sig << (8 * j);
        const double step = (double)s * e4m3_value(sig);  // exact: 24-bit times 4-bit
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          int q = 0;
          if (step != 0.0) {
            q = __double2int_rn(__ddiv_rn(v[16 * j + i], step));
            q = q > F::kQmax ? F::kQmax : (q < -F::kQmax ? -F::kQmax : q);
          }
          const uint32_t u = (uint32_t)(q + F::kBias);
          const int k = 16 * j + i;  // code index in the k-block
          const int word = k >> 3, pos = (k & 7) >> 1, upper = k & 1;
          lo[word] |= (u & 15u) << (16 * upper + 4 * pos);
          if (BITS == 6) {
            const int hword = k >> 4, hpos = (k & 15) >> 1;
            hi[hword] |= (u >> 4) << (16 * upper + 2 * hpos);
          }
        }
      }
      uint8_t* tile = out + (rb * kbs + kb) * (int64_t)F::kTileBytes;
      *reinterpret_cast<uint4*>(tile + r * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(tile + 2048 + r * 16) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
      if (BITS == 6)
        *reinterpret_cast<uint4*>(tile + 4096 + r * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint32_t*>(tile + F::kScaleOff + r * 4) = sig_word;
    }
    if (tid == 0) row_scale[row] = s;
    __syncthreads();  // the row buffer and red[] are reused by the next row
  }
}

// ----------------------------------------------------------------- GEMM ----
enum LowbitEpilogue : int {
  kLbF32 = 0,     // out fp32 [G, M, N]: the accumulator acc = sum_k x * sigma * q
  kLbBf16 = 1,    // out bf16 [G, M, N]: y = acc * (s_x * s_r)
  kLbSwiglu = 2   // out fp32 [G, M, F]: h = silu(y[:, f]) * y[:, F + f], N = 2F
};

namespace lb {
constexpr int kMaxRawStages = 16;  // packed weights + int8 activation codes, per K-step of 64
constexpr int kCvStages = 4;       // decoded: A in TMEM (64 columns), B in shared memory
constexpr int kMaxNt = 128;        // tokens per tile
constexpr int kConvGroups = 4;     // = kCvStages: group g decodes the K-steps j with j % 4 == g
constexpr int kConvWarps = 4 * kConvGroups;  // one warp per TMEM lane quadrant in each group
constexpr int kEpiWarps = 4;
constexpr int kMmaWarps = 4;      // MMA issuers: one per accumulator (2 blocks x ks sets)
constexpr int kConvWarp0 = 1 + kMmaWarps;
constexpr int kEpiWarp0 = kConvWarp0 + kConvWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr uint32_t kTmemCols = 512;
constexpr int kAccCol0 = kCvStages * 64;  // accumulators after the A stages
constexpr int kBarBytes = 512;
constexpr int kSmemMax = 232448;          // the opt-in limit per CTA
// Shared memory of one raw stage for nt tokens (the two weight tiles, then
// the activation box), rounded to 1024 bytes.
template <int BITS>
__host__ __device__ constexpr int raw_stage_bytes(int nt) {
  return (2 * LbFmt<BITS>::kTileBytes + nt * 64 + 1023) / 1024 * 1024;
}
// As many raw stages as fit beside the decoded-B ring (the weight stream is
// compressed, so a deep ring is what keeps enough bytes in flight).
template <int BITS>
__host__ __device__ constexpr int raw_stages(int nt) {
  const int room = kSmemMax - 1024 - kBarBytes - kCvStages * nt * 128;
  const int r = room / raw_stage_bytes<BITS>(nt);
  return r > kMaxRawStages ? kMaxRawStages : r;
}
template <int BITS>
__host__ __device__ constexpr int smem_bytes(int nt) {
  return raw_stages<BITS>(nt) * raw_stage_bytes<BITS>(nt) + kCvStages * nt * 128 + kBarBytes +
         1024;
}
static_assert(raw_stages<6>(kMaxNt) >= 6 && smem_bytes<6>(kMaxNt) <= kSmemMax, "shared memory");
}  // namespace lb

struct LowbitArgs {
  int G, M, N, K;       // groups, tokens per group, weight rows per group (2F for SwiGLU), K
  int n_out;            // output columns: N, or F for SwiGLU
  int nt;               // tokens per tile: a multiple of 16, at most 128
  int box_rows;         // rows of the activation box: min(nt, M)
  int t_blocks, w_blocks, k_blocks, num_tiles;
  int n_acc;            // accumulator buffers (1 or 2)
  int ks;               // accumulator sets per weight block (1, 2 or 4): K-slice k of every
                        // K-step accumulates into set k % ks, and the epilogue adds the
                        // sets; consecutive MMAs then write different accumulators, so
                        // their latency overlaps (small-N MMAs into one accumulator
                        // serialise on it). 2 * ks * nt * n_acc <= 256 columns.
  int raw_stages;       // depth of the raw ring (lb::raw_stages)
  const uint8_t* wq;    // packed weight tiles (see the top of this file)
  const float* s_w;     // [G*N] row scales
  const float* s_x;     // [G*M] token scales
  void* out;
};

// fp16x2 helpers on raw bits
__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// two E4M3 bytes (low byte -> low half) to an fp16 pair, exactly
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
  uint32_t d;
  const unsigned short s = (unsigned short)two;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(s));
  return d;
}

// Four int8 codes to two fp16 pairs, exactly: the byte u = x + 128 under the
// fp16 pattern of 1024 (0x64 high byte) is 1024 + u; minus 1152 leaves x.
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  lo = h2_sub(__byte_perm(u, 0x64646464u, 0x4140), 0x64806480u);
  hi = h2_sub(__byte_perm(u, 0x64646464u, 0x4342), 0x64806480u);
}

// Row r's half (32 codes, two groups) of one k-block of a weight tile, decoded
// to 16 fp16 pairs q * sigma / 16 in K order.
template <int BITS>
__device__ __forceinline__ void lb_decode_row(const uint8_t* tile, int r, int half,
                                              uint32_t (&o)[16]) {
  using F = LbFmt<BITS>;
  const uint4 lw = *reinterpret_cast<const uint4*>(tile + half * 2048 + r * 16);
  uint2 hw = make_uint2(0u, 0u);
  if (BITS == 6) hw = *reinterpret_cast<const uint2*>(tile + 4096 + r * 16 + half * 8);
  const uint32_t sw = *reinterpret_cast<const uint32_t*>(tile + F::kScaleOff + r * 4);
  const uint32_t sp = h2_mul(e4m3x2_to_h2(sw >> (16 * half)), 0x2C002C00u);  // sigma / 16
  const uint32_t s_a = __byte_perm(sp, 0u, 0x1010), s_b = __byte_perm(sp, 0u, 0x3232);
  const uint32_t c_a = h2_mul(s_a, F::kNegMagic2), c_b = h2_mul(s_b, F::kNegMagic2);
  const uint32_t w[4] = {lw.x, lw.y, lw.z, lw.w};
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const uint32_t s = ii < 2 ? s_a : s_b, c = ii < 2 ? c_a : c_b;
    const uint32_t hword = ii < 2 ? hw.x : hw.y;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t t = ((w[ii] >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
      if (BITS == 6) t |= ((hword >> (2 * (4 * (ii & 1) + j))) & 0x00030003u) << 4;
      o[4 * ii + j] = h2_fma(t, s, c);
    }
  }
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}


// generic-proxy shared-memory writes made visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Instruction descriptor: f32 accumulator (bits 4-5 = 1), f16 A and B (bits
// 7-9 and 10-12 = 0), both K-major, N>>3 at bits 17-22, M>>4 at 24-28.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]^T, f16 x f16 -> f32, issued by one thread.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void lb_decode_tile(const LowbitArgs& a, int tile, int& g, int& wb,
                                               int& tb) {
  tb = tile % a.t_blocks;
  const int rest = tile / a.t_blocks;
  wb = rest % a.w_blocks;
  g = rest / a.w_blocks;
}

// The two weight row blocks of tile (g, wb): SwiGLU the gate block wb and the
// matching up block, otherwise row blocks 2wb and 2wb + 1.
__device__ __forceinline__ int64_t lb_row_block(const LowbitArgs& a, int g, int wb, int which,
                                                bool swiglu) {
  const int64_t base = (int64_t)g * (a.N / 128);
  return swiglu ? base + wb + (which ? a.n_out / 128 : 0) : base + 2 * wb + which;
}

// One persistent CTA per SM. Tiles (group, weight block of 2 x 128 rows,
// token block of nt), token block fastest so CTAs running together share the
// weight tiles through L2.
//   warp 0      producer: per K-step one bulk copy per weight tile and a 3-D
//               TMA box {64 codes, box_rows tokens} of the activation codes
//   warps 1-4   MMA issuers (warp 1 also allocates 512 TMEM columns): one
//               lane each issues tcgen05.mma kind::f16 M=128 N=nt K=16 (A
//               from TMEM) into its own accumulator (weight block, set);
//               2 * ks of them are active
//   warps 5-20  converters in four groups of four warps; group g takes the
//               K-steps j with j % 4 == g (decoded stage g), so four K-steps
//               are decoded at once: warp w decodes the rows of TMEM lane
//               quadrant w % 4 of both weight blocks into the A stage
//               (tcgen05.st) and widens a quarter of the activation codes to
//               the fp16 B stage (one K-step's decode is a chain of dependent
//               loads, conversions and tensor-memory stores: several in
//               flight keep the tensor cores fed)
//   warps 21-24 epilogue: tcgen05.ld of the quadrant's rows, 16 tokens at a
//               time; lanes hold consecutive weight rows, so each token's
//               outputs are one contiguous store per warp
template <int BITS, int EPI>
__global__ void __launch_bounds__(lb::kThreads, 1)
    gemm_lowbit_tcgen05_kernel(const __grid_constant__ CUtensorMap tmX, const LowbitArgs args) {
  using F = LbFmt<BITS>;
  constexpr int S = lb::kCvStages;
  constexpr bool kSwiglu = EPI == kLbSwiglu;
  const int nt = args.nt;
  const int R = args.raw_stages;
  const int RAW = lb::raw_stage_bytes<BITS>(nt);
  const int BST = nt * 128;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t rawp = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((rawp + 1023u) & ~1023u) - rawp);
  uint8_t* raw = smem;
  uint8_t* bst = smem + R * RAW;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bst + S * BST);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = bars + lb::kMaxRawStages;
  uint64_t* cv_full = bars + 2 * lb::kMaxRawStages;
  uint64_t* cv_empty = cv_full + S;
  uint64_t* tfull = cv_empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;  // one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + lb::kMmaWarps);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], 4);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&cv_full[s], 4);
      mbar_init(&cv_empty[s], 2 * args.ks);   // every issuer commits
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 2 * args.ks);
      mbar_init(&tempty[a], lb::kEpiWarps);
    }
    for (int i = 0; i < lb::kMmaWarps; ++i) mbar_init(&drain[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == 1) {
    tmem_alloc(tmem_slot, lb::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  uint32_t issued_mask = 0, issued_parity = 0;
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      const uint32_t tx = (uint32_t)(2 * F::kTileBytes + args.box_rows * 64);
      auto load_w = [&](int s, int g, int wb, int kb) {
        uint8_t* dst = raw + s * RAW;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const int64_t rb = lb_row_block(args, g, wb, which, kSwiglu);
          bulk_load_1d(dst + which * F::kTileBytes,
                       args.wq + (rb * args.k_blocks + kb) * (int64_t)F::kTileBytes,
                       (uint32_t)F::kTileBytes, &raw_full[s], pol_w);
        }
      };
      auto load_x = [&](int s, int g, int tb, int kb) {
        tma_load_3d(raw + s * RAW + 2 * F::kTileBytes, &tmX, &raw_full[s], kb * 64, tb * nt, g,
                    pol_x);
      };
      // the first tile's first stages: weights before the wait for the kernel
      // that wrote the activation codes (they do not depend on it)
      int pre = 0;
      if ((int)blockIdx.x < args.num_tiles) {
        int g, wb, tb;
        lb_decode_tile(args, blockIdx.x, g, wb, tb);
        pre = min(args.k_blocks, R);
        for (int kb = 0; kb < pre; ++kb) {
          mbar_arrive_expect_tx(&raw_full[kb], tx);
          load_w(kb, g, wb, kb);
        }
        griddep_wait();
        for (int kb = 0; kb < pre; ++kb) {
          load_x(kb, g, tb, kb);
          issued_mask |= 1u << kb;
        }
      } else {
        griddep_wait();
      }
      int s = pre % R;
      uint32_t ph = pre == R ? 1u : 0u;
      for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x) {
        int g, wb, tb;
        lb_decode_tile(args, tile, g, wb, tb);
        bool ok = true;
        for (int kb = tile == (int)blockIdx.x ? pre : 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(&raw_empty[s], ph ^ 1u, abort_flag, kErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&raw_full[s], tx);
          load_w(s, g, wb, kb);
          load_x(s, g, tb, kb);
          issued_mask |= 1u << s;
          issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
          if (++s == R) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp < lb::kConvWarp0) {
    // MMA issuers: issuer i owns accumulator (block i / ks, set i % ks) and
    // issues its MMAs (the K-slices k of every K-step with k % ks == i % ks).
    // A thread waits about 120 cycles on every tcgen05.mma it issues (measured
    // on B200, independent of N up to 128), so short MMAs need several
    // issuers to keep the tensor pipe busy; they write different
    // accumulators, so their order does not matter.
    const int issuer = warp - 1;
    const int ks = args.ks;
    if (lane == 0 && issuer < 2 * ks) {
      const int b = issuer / ks, q = issuer % ks;
      const uint32_t idesc = idesc_f16_f32(128, nt);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x, ++it) {
        const int acc = args.n_acc == 2 ? (it & 1) : 0;
        const uint32_t acc_phase = (uint32_t)(args.n_acc == 2 ? (it >> 1) : it) & 1u;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, kErrTimeoutTmemEmpty)) break;
        tc_fence_after();
        // accumulator (block b, set q) at column base + (b * ks + q) * nt
        const uint32_t d = tmem_base + (uint32_t)(lb::kAccCol0 + acc * 2 * ks * nt +
                                                  (b * ks + q) * nt);
        bool ok = true;
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(&cv_full[s], ph, abort_flag, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_addr = smem_u32(bst + s * BST);
          const uint32_t a_col = tmem_base + (uint32_t)(s * 64 + b * 32);
          for (int k = q; k < 4; k += ks) {
            const uint32_t accum = (kb > 0 || k >= ks) ? 1u : 0u;
            umma_f16_ts(d, a_col + 8 * k, sdesc_k_sw128(b_addr + 32 * k), idesc, accum);
          }
          mma_issued = true;
          umma_commit(&cv_empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
    }
  } else if (warp < lb::kEpiWarp0) {
    // ---------------------------------------------------------- converters --
    const int cg = (warp - lb::kConvWarp0) >> 2;   // group = decoded stage
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int ct = ((warp - lb::kConvWarp0) & 3) * 32 + lane;
    const uint32_t t_lane = (uint32_t)(quad * 32) << 16;
    const int my_tiles = (int)blockIdx.x < args.num_tiles
                             ? (args.num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                             : 0;
    const int steps = my_tiles * args.k_blocks;
    const uint32_t tcol = tmem_base + t_lane + (uint32_t)(cg * 64);
    uint8_t* bt = bst + cg * BST;
    for (int j = cg; j < steps; j += lb::kConvGroups) {
      const int rs = j % R;
      bool w_ok = mbar_wait(&raw_full[rs], (uint32_t)(j / R) & 1u, abort_flag, kErrTimeoutFull);
      w_ok = w_ok && mbar_wait(&cv_empty[cg], ((uint32_t)(j / lb::kConvGroups) & 1u) ^ 1u,
                               abort_flag, kErrTimeoutEmpty);
      if (__any_sync(0xffffffffu, !w_ok)) break;
      const uint8_t* st = raw + rs * RAW;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t a[16];
          lb_decode_row<BITS>(st + which * F::kTileBytes, r, half, a);
          tmem_st16(tcol + (uint32_t)(which * 32 + half * 16), a);
        }
      }
      const uint8_t* act = st + 2 * F::kTileBytes;
      for (int u = ct; u < nt * 8; u += 128) {
        const int row = u >> 3, ch = u & 7;
        const uint2 xv = *reinterpret_cast<const uint2*>(act + row * 64 + ch * 8);
        uint4 o;
        i8x4_to_h2x2(xv.x, o.x, o.y);
        i8x4_to_h2x2(xv.y, o.z, o.w);
        *reinterpret_cast<uint4*>(bt + row * 128 + ((ch ^ (row & 7)) << 4)) = o;
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&cv_full[cg]);
        mbar_arrive(&raw_empty[rs]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    griddep_wait();  // the token scales come from the previous kernel
    griddep_launch_dependents();
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t t_lane = (uint32_t)(quad * 32) << 16;
    const int ks = args.ks;
    int it = 0;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x, ++it) {
      const int acc = args.n_acc == 2 ? (it & 1) : 0;
      const uint32_t acc_phase = (uint32_t)(args.n_acc == 2 ? (it >> 1) : it) & 1u;
      // the tile's scales are requested before the wait for its accumulators:
      // lane l holds the token scales of tokens t0 + l + 32 i
      int g, wb, tb;
      lb_decode_tile(args, tile, g, wb, tb);
      const int t0 = tb * nt;
      const int n0 = kSwiglu ? wb * 128 + r : wb * 256 + r;
      const int n1 = kSwiglu ? args.n_out + n0 : n0 + 128;
      const float sw0 = __ldg(args.s_w + (int64_t)g * args.N + n0);
      const float sw1 = __ldg(args.s_w + (int64_t)g * args.N + n1);
      static_assert(lb::kMaxNt == 128, "four token-scale registers per lane");
      auto sx_at = [&](int i) {
        const int t = t0 + 32 * i + lane;
        return (EPI != kLbF32 && 32 * i < nt && t < args.M)
                   ? __ldg(args.s_x + (int64_t)g * args.M + t) : 0.0f;
      };
      const float sx0 = sx_at(0), sx1 = sx_at(1), sx2 = sx_at(2), sx3 = sx_at(3);
      const bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, kErrTimeoutTmemFull);
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const uint32_t dbase = tmem_base + t_lane + (uint32_t)(lb::kAccCol0 + acc * 2 * ks * nt);
      for (int c0 = 0; c0 < nt; c0 += 16) {
        // each block's accumulator sets, added in set order
        float v0[16], v1[16];
        {
          uint32_t u0[16], u1[16];
          tmem_ld16(dbase + c0, u0);
          tmem_ld16(dbase + (uint32_t)(ks * nt) + c0, u1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v0[i] = __uint_as_float(u0[i]);
            v1[i] = __uint_as_float(u1[i]);
          }
        }
        for (int q = 1; q < ks; ++q) {
          uint32_t u[16];
          tmem_ld16(dbase + (uint32_t)(q * nt) + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v0[i] = __fadd_rn(v0[i], __uint_as_float(u[i]));
          tmem_ld16(dbase + (uint32_t)((ks + q) * nt) + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v1[i] = __fadd_rn(v1[i], __uint_as_float(u[i]));
        }
        // the register holding this chunk's token scales
        const float sx_src = c0 < 32 ? sx0 : c0 < 64 ? sx1 : c0 < 96 ? sx2 : sx3;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = t0 + c0 + i;
          const float sx = __shfl_sync(0xffffffffu, sx_src, (c0 & 16) + i);
          if (t >= args.M) continue;
          const float a0 = __fmul_rn(v0[i], 16.0f);
          const float a1 = __fmul_rn(v1[i], 16.0f);
          const int64_t orow = (int64_t)g * args.M + t;
          if constexpr (EPI == kLbF32) {
            float* out = reinterpret_cast<float*>(args.out) + orow * args.N;
            out[n0] = a0;
            out[n1] = a1;
          } else if constexpr (EPI == kLbBf16) {
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(args.out) + orow * args.N;
            out[n0] = __float2bfloat16_rn(__fmul_rn(a0, __fmul_rn(sx, sw0)));
            out[n1] = __float2bfloat16_rn(__fmul_rn(a1, __fmul_rn(sx, sw1)));
          } else {
            const float yg = __fmul_rn(a0, __fmul_rn(sx, sw0));
            const float yu = __fmul_rn(a1, __fmul_rn(sx, sw1));
            reinterpret_cast<float*>(args.out)[orow * args.n_out + n0] =
                __fmul_rn(silu_f32(yg), yu);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // after a timeout: let every issued copy and MMA land before the shared
    // memory and the TMEM columns are released
    int never = 0;
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < R; ++s)
        if (issued_mask & (1u << s))
          mbar_wait_limit(&raw_full[s], (issued_parity >> s) & 1u, &never, kErrTimeoutTeardown,
                          100000000ull);
    }
    if (warp >= 1 && warp < lb::kConvWarp0 && lane == 0 && mma_issued) {
      umma_commit(&drain[warp - 1]);
      mbar_wait_limit(&drain[warp - 1], 0, &never, kErrTimeoutTeardown, 100000000ull);
    }
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, lb::kTmemCols);
  }
}

}  // namespace convrot
