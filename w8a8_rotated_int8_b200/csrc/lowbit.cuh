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
// (at most 9 significant bits, between 2^-13 and 28 * 31). Converter warps
// decode the weights into shared memory as the N = 256 operand (two 128-row
// blocks, the 128-byte swizzle) and widen the activation codes into the M
// operand (the tile's tokens), so every MMA has N = 256 whatever the token
// count: a thread issuing tcgen05.mma waits about 120 cycles per instruction
// (measured on B200) whether N is 16 or 128, so short instructions cannot
// keep the tensor core busy. M is 64 for tiles of up to 64 tokens, 128 up to
// 128, and 256 over a CTA pair for more (each CTA then decodes one of the two
// weight blocks). D[token, weight row] accumulates sum_k x * q * sigma / 16;
// the epilogue multiplies by 16 (exact) and dequantises y = acc * (s_x * s_r).
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
constexpr int kMaxRawStages = 8;        // packed weights + int8 activation codes, per K-step of 64
constexpr int kConvGroups = 3;          // group g decodes the K-steps j with j % 3 == g
constexpr int kConvWarps = 4 * kConvGroups;
constexpr int kEpiWarps = 4;
constexpr int kConvWarp0 = 2;
constexpr int kEpiWarp0 = kConvWarp0 + kConvWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kMaxNt = 128;             // tokens per tile (per CTA of a pair)
constexpr int kABytes = kMaxNt * 128;   // widened tokens: 128 rows x 64 codes, fp16
constexpr uint32_t kTmemCols = 512;     // two accumulators of 256 columns
constexpr int kBarBytes = 512;
constexpr int kSmemMax = 232448;        // the opt-in limit per CTA
// A CTA decodes both 128-row weight blocks of a tile, or (CTA pair) one.
__host__ __device__ constexpr int w_tiles(bool pair) { return pair ? 1 : 2; }
// decoded stages: fp16 weights (the N operand, this CTA's rows) and tokens
__host__ __device__ constexpr int dec_stages(bool pair) { return pair ? 4 : 3; }
__host__ __device__ constexpr int b_bytes(bool pair) { return w_tiles(pair) * 128 * 128; }
__host__ __device__ constexpr int dec_bytes(bool pair) { return b_bytes(pair) + kABytes; }
// Shared memory of one raw stage for nt tokens (this CTA's weight tiles, then
// the activation box), rounded to 1024 bytes.
template <int BITS>
__host__ __device__ constexpr int raw_stage_bytes(int nt, bool pair) {
  return (w_tiles(pair) * LbFmt<BITS>::kTileBytes + nt * 64 + 1023) / 1024 * 1024;
}
// As many raw stages as fit beside the decoded stages.
template <int BITS>
__host__ __device__ constexpr int raw_stages(int nt, bool pair) {
  const int room = kSmemMax - 1024 - kBarBytes - dec_stages(pair) * dec_bytes(pair);
  const int r = room / raw_stage_bytes<BITS>(nt, pair);
  return r > kMaxRawStages ? kMaxRawStages : r;
}
template <int BITS>
__host__ __device__ constexpr int smem_bytes(int nt, bool pair) {
  return dec_stages(pair) * dec_bytes(pair) +
         raw_stages<BITS>(nt, pair) * raw_stage_bytes<BITS>(nt, pair) + kBarBytes + 1024;
}
static_assert(raw_stages<6>(kMaxNt, false) >= 3 && smem_bytes<6>(kMaxNt, false) <= kSmemMax,
              "shared memory");
static_assert(raw_stages<6>(kMaxNt, true) >= 4 && smem_bytes<6>(kMaxNt, true) <= kSmemMax,
              "shared memory");
}  // namespace lb

struct LowbitArgs {
  int G, M, N, K;       // groups, tokens per group, weight rows per group (2F for SwiGLU), K
  int n_out;            // output columns: N, or F for SwiGLU
  int nt;               // tokens per tile (per CTA): a multiple of 16, at most 128
                        // (128 for CTA pairs, whose tiles hold 2 x 128 tokens)
  int box_rows;         // rows of the activation box: min(nt, M)
  int t_blocks, w_blocks, k_blocks, num_tiles;  // token blocks of the tile's tokens
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

// Half `half` (32 codes, two groups) of one row of a weight tile's k-block,
// from the row's words (lw: the half's plane, hw: its top-bit words for six
// bits, sw: the row's four E4M3 group scales), to 16 fp16 pairs
// q * sigma / 16 in K order.
template <int BITS>
__device__ __forceinline__ void lb_decode_words(uint4 lw, uint2 hw, uint32_t sw, int half,
                                                uint32_t (&o)[16]) {
  using F = LbFmt<BITS>;
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

// generic-proxy shared-memory writes made visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Instruction descriptor: f32 accumulator (bits 4-5 = 1), f16 A and B (bits
// 7-9 and 10-12 = 0), both K-major, N>>3 at bits 17-22, M>>4 at 24-28.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, f16 x f16 -> f32, issued by one thread.
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The CTA-pair form: D (M = 256 over the pair) (+)= A * B^T, each CTA
// supplying its 128 token rows of A and its 128 of the N = 256 weight rows of
// B at the same shared-memory offsets; issued by one thread of the leader.
__device__ __forceinline__ void umma_f16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
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

// One persistent CTA per SM, or (PAIR) one CTA pair per two SMs. A tile is
// (group, weight block of 2 x 128 rows, token block), the token block fastest
// so CTAs running together share the weight tiles through L2. A single CTA
// takes nt tokens and decodes both weight blocks; the two CTAs of a pair take
// 128 tokens each and decode one weight block each (the gate / first block in
// the leader, rank 0), and the leader's MMAs (M = 256 over the pair) read
// both CTAs' halves, so each decoded weight serves 256 tokens.
//   warp 0      producer: per K-step one bulk copy per weight tile and a 3-D
//               TMA box {64 codes, box_rows tokens} of the activation codes,
//               into this CTA's shared memory
//   warp 1      allocates 512 TMEM columns (in both CTAs of a pair); one lane
//               (of the leader) issues tcgen05.mma kind::f16 with N = 256 and
//               K = 16, four per K-step, into one of two 256-column
//               accumulators; in the other CTA of a pair, lanes 0..S-1 relay
//               its decoded stages' completion to the leader
//   warps 2-13  converters in three groups of four warps; group g takes the
//               K-steps j with j % 3 == g: thread i decodes row i of each of
//               the CTA's weight tiles into the N operand and widens a share
//               of the activation codes into the M operand, in decoded stage
//               j % S
//   warps 14-17 epilogue: tcgen05.ld of the quadrant's token rows, 16
//               columns at a time; each lane writes its row's outputs
// M64 (single CTA, at most 64 tokens per tile): M = 64 instructions, half
// the tensor work and half the token operand read per instruction.
template <int BITS, int EPI, bool PAIR, bool M64>
__global__ void __launch_bounds__(lb::kThreads, 1)
    gemm_lowbit_tcgen05_kernel(const __grid_constant__ CUtensorMap tmX, const LowbitArgs args) {
  using F = LbFmt<BITS>;
  constexpr int S = lb::dec_stages(PAIR);
  constexpr int WT = lb::w_tiles(PAIR);
  constexpr int DEC = lb::dec_bytes(PAIR);
  constexpr bool kSwiglu = EPI == kLbSwiglu;
  const int nt = args.nt;
  const int R = args.raw_stages;
  const int RAW = lb::raw_stage_bytes<BITS>(nt, PAIR);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t rawp = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((rawp + 1023u) & ~1023u) - rawp);
  uint8_t* dec = smem;                               // S x (B, then A 16 KB)
  uint8_t* raw = smem + S * DEC;                     // R raw stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw + R * RAW);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = bars + lb::kMaxRawStages;
  uint64_t* cv_full = bars + 2 * lb::kMaxRawStages;
  uint64_t* cv_empty = cv_full + S;
  uint64_t* tfull = cv_empty + S;
  uint64_t* tempty = tfull + 2;                      // the leader's, for a pair
  uint64_t* drain = tempty + 2;
  uint64_t* fin = drain + 1;                         // pair teardown handshake
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // CTA or pair
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // this CTA's first token row within a tile's token block
  const int row0 = PAIR ? (int)rank * lb::kMaxNt : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], 4);
    }
    for (int s = 0; s < S; ++s) {
      // a pair's leader: its four converter warps and the other CTA's relay
      mbar_init(&cv_full[s], PAIR && leader ? 5 : 4);
      mbar_init(&cv_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], (PAIR ? 2 : 1) * lb::kEpiWarps);
    }
    mbar_init(drain, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, lb::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, lb::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // both CTAs' barriers exist before any remote use
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  uint32_t issued_mask = 0, issued_parity = 0;
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      const uint32_t tx = (uint32_t)(WT * F::kTileBytes + args.box_rows * 64);
      auto load_w = [&](int s, int g, int wb, int kb) {
        uint8_t* dst = raw + s * RAW;
#pragma unroll
        for (int i = 0; i < WT; ++i) {
          const int64_t rb = lb_row_block(args, g, wb, PAIR ? (int)rank : i, kSwiglu);
          bulk_load_1d(dst + i * F::kTileBytes,
                       args.wq + (rb * args.k_blocks + kb) * (int64_t)F::kTileBytes,
                       (uint32_t)F::kTileBytes, &raw_full[s], pol_w);
        }
      };
      const int tb_rows = PAIR ? 2 * lb::kMaxNt : nt;  // tokens per token block
      auto load_x = [&](int s, int g, int tb, int kb) {
        tma_load_3d(raw + s * RAW + WT * F::kTileBytes, &tmX, &raw_full[s], kb * 64,
                    tb * tb_rows + row0, g, pol_x);
      };
      // the first tile's first stages: weights before the wait for the kernel
      // that wrote the activation codes (they do not depend on it)
      int pre = 0;
      if (unit < args.num_tiles) {
        int g, wb, tb;
        lb_decode_tile(args, unit, g, wb, tb);
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
      for (int tile = unit; tile < args.num_tiles; tile += n_units) {
        int g, wb, tb;
        lb_decode_tile(args, tile, g, wb, tb);
        bool ok = true;
        for (int kb = tile == unit ? pre : 0; kb < args.k_blocks; ++kb) {
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
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_f16_f32(PAIR ? 256 : M64 ? 64 : 128, 256);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int tile = unit; tile < args.num_tiles; tile += n_units, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait<PAIR>(&tempty[acc], acc_phase ^ 1u, abort_flag, kErrTimeoutTmemEmpty))
          break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * 256);
        bool ok = true;
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait<PAIR>(&cv_full[s], ph, abort_flag, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_addr = smem_u32(dec + s * DEC);
          const uint32_t a_addr = b_addr + lb::b_bytes(PAIR);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sdesc_k_sw128(a_addr + 32 * k);
            const uint64_t bd = sdesc_k_sw128(b_addr + 32 * k);
            if constexpr (PAIR)
              umma_f16_ss_pair(d, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            else
              umma_f16_ss(d, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_issued = true;
          if constexpr (PAIR)
            umma_commit_pair(&cv_empty[s], 0x3);
          else
            umma_commit(&cv_empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (PAIR)
          umma_commit_pair(&tfull[acc], 0x3);
        else
          umma_commit(&tfull[acc]);
      }
    } else if (PAIR && !leader && lane < S) {
      // relay of the other CTA: lane s passes each completed phase of this
      // CTA's decoded stage s on to the leader's barrier of that stage, off
      // the converters' path. The converters' shared-memory writes are
      // complete (and fenced for the async proxy) once the local phase has
      // completed; the relay observes that before it arrives, and the
      // leader's MMAs, issued after the leader observes the arrive, read
      // this CTA's shared memory directly. The arrive is relaxed: a release
      // at cluster scope costs about a microsecond per K-step here (measured:
      // 287 against 222 us for a 64 x 3072 x 2048 x 256-token GEMM).
      const int my_tiles =
          unit < args.num_tiles ? (args.num_tiles - 1 - unit) / n_units + 1 : 0;
      const int steps = my_tiles * args.k_blocks;
      const uint32_t remote = mapa_shared(smem_u32(&cv_full[lane]), 0);
      for (int j = lane; j < steps; j += S) {
        if (!mbar_wait(&cv_full[lane], (uint32_t)(j / S) & 1u, abort_flag, kErrTimeoutFull)) break;
        mbar_arrive_cluster_relaxed(remote);
      }
    }
  } else if (warp < lb::kEpiWarp0) {
    // ---------------------------------------------------------- converters --
    const int cg = (warp - lb::kConvWarp0) >> 2;
    const int ti = ((warp - lb::kConvWarp0) & 3) * 32 + lane;  // 0..127
    const int my_tiles =
        unit < args.num_tiles ? (args.num_tiles - 1 - unit) / n_units + 1 : 0;
    const int steps = my_tiles * args.k_blocks;
    for (int j = cg; j < steps; j += lb::kConvGroups) {
      const int rs = j % R;
      const int ds = j % S;
      uint8_t* bt = dec + ds * DEC;        // weights: WT x 128 rows x 128 bytes
      uint8_t* at = bt + lb::b_bytes(PAIR);  // tokens: rows 0..nt-1 x 128 bytes
      const bool r_ok =
          mbar_wait(&raw_full[rs], (uint32_t)(j / R) & 1u, abort_flag, kErrTimeoutFull);
      if (__any_sync(0xffffffffu, !r_ok)) break;
      // the K-step's words into registers, then the raw stage goes back to
      // the producer: its next copy is in flight while this group decodes
      const uint8_t* st = raw + rs * RAW;
      uint4 lw[WT][2];
      uint2 hw[WT][2];
      uint32_t sw[WT];
#pragma unroll
      for (int i = 0; i < WT; ++i) {
        const uint8_t* tile = st + i * F::kTileBytes;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          lw[i][half] = *reinterpret_cast<const uint4*>(tile + half * 2048 + ti * 16);
          hw[i][half] =
              BITS == 6 ? *reinterpret_cast<const uint2*>(tile + 4096 + ti * 16 + half * 8)
                        : make_uint2(0u, 0u);
        }
        sw[i] = *reinterpret_cast<const uint32_t*>(tile + F::kScaleOff + ti * 4);
      }
      constexpr int kXChunks = lb::kMaxNt * 8 / 128;  // 8-byte chunks of codes per thread
      uint2 xv[kXChunks];
      const uint8_t* act = st + WT * F::kTileBytes;
#pragma unroll
      for (int m = 0; m < kXChunks; ++m) {
        const int u = ti + 128 * m;
        xv[m] = u < nt * 8 ? *reinterpret_cast<const uint2*>(act + u * 8) : make_uint2(0u, 0u);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&raw_empty[rs]);
      const bool d_ok =
          mbar_wait(&cv_empty[ds], ((uint32_t)(j / S) & 1u) ^ 1u, abort_flag, kErrTimeoutEmpty);
      if (__any_sync(0xffffffffu, !d_ok)) break;
#pragma unroll
      for (int i = 0; i < WT; ++i) {
        const int row = i * 128 + ti;
        uint8_t* dst = bt + row * 128;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[16];
          lb_decode_words<BITS>(lw[i][half], hw[i][half], sw[i], half, o);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(dst + (((4 * half + c) ^ (row & 7)) << 4)) =
                make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        }
      }
#pragma unroll
      for (int m = 0; m < kXChunks; ++m) {
        const int u = ti + 128 * m;
        if (u < nt * 8) {
          const int row = u >> 3, ch = u & 7;
          uint4 o;
          i8x4_to_h2x2(xv[m].x, o.x, o.y);
          i8x4_to_h2x2(xv[m].y, o.z, o.w);
          *reinterpret_cast<uint4*>(at + row * 128 + ((ch ^ (row & 7)) << 4)) = o;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&cv_full[ds]);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    griddep_wait();  // the token scales come from the previous kernel
    griddep_launch_dependents();
    const int quad = warp & 3;
    const uint32_t t_lane = (uint32_t)(quad * 32) << 16;
    const int tb_rows = PAIR ? 2 * lb::kMaxNt : nt;
    int it = 0;
    for (int tile = unit; tile < args.num_tiles; tile += n_units, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      int g, wb, tb;
      lb_decode_tile(args, tile, g, wb, tb);
      // column j of the accumulator is weight row j of the tile's two blocks;
      // every lane reads the same scales (one broadcast load per warp)
      const float* sw0 = args.s_w + (int64_t)g * args.N + (kSwiglu ? wb * 128 : wb * 256);
      const float* sw1 = kSwiglu ? sw0 + args.n_out : sw0 + 128;
      const int t0 = tb * tb_rows + row0;   // this CTA's first token
      // M = 64: accumulator row r sits in lane 16 of sub-partition r / 16's
      // 32 lanes plus r % 16, so lanes 16..31 of each warp hold no row
      constexpr int kRowsPerQuad = M64 ? 16 : 32;
      const int row = quad * kRowsPerQuad + (lane & (kRowsPerQuad - 1));
      const int t = t0 + row;
      const bool valid = lane < kRowsPerQuad && row < nt && t < args.M;
      const float sx = (EPI != kLbF32 && valid) ? __ldg(args.s_x + (int64_t)g * args.M + t) : 0.0f;
      const bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, kErrTimeoutTmemFull);
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + t_lane + (uint32_t)(acc * 256);
      const bool warp_rows =
          quad * kRowsPerQuad < nt && t0 + quad * kRowsPerQuad < args.M;  // warp-uniform
      if (warp_rows) {
        const int64_t orow = (int64_t)g * args.M + t;
        if constexpr (kSwiglu) {
          float* out = reinterpret_cast<float*>(args.out) + orow * args.n_out + wb * 128;
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            __syncwarp();
            uint32_t gv[16], uv[16];
            tmem_ld16(d + c * 16, gv);
            tmem_ld16(d + 128 + c * 16, uv);
            float sg[16], su[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              *reinterpret_cast<float4*>(sg + 4 * q) =
                  __ldg(reinterpret_cast<const float4*>(sw0 + c * 16) + q);
              *reinterpret_cast<float4*>(su + 4 * q) =
                  __ldg(reinterpret_cast<const float4*>(sw1 + c * 16) + q);
            }
            tmem_wait_ld();
            float h[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float yg =
                  __fmul_rn(__fmul_rn(__uint_as_float(gv[i]), 16.0f), __fmul_rn(sx, sg[i]));
              const float yu =
                  __fmul_rn(__fmul_rn(__uint_as_float(uv[i]), 16.0f), __fmul_rn(sx, su[i]));
              h[i] = __fmul_rn(silu_f32(yg), yu);
            }
            if (valid) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4*>(out + c * 16 + 4 * q) =
                    make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
            }
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            __syncwarp();
            uint32_t v[16];
            tmem_ld16(d + c * 16, v);
            float sc[16];
            if constexpr (EPI == kLbBf16) {
              const float* sp = (c < 8 ? sw0 : sw1) + (c & 7) * 16;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4*>(sc + 4 * q) =
                    __ldg(reinterpret_cast<const float4*>(sp) + q);
            }
            tmem_wait_ld();
            if (valid) {
              const int n0 = wb * 256 + c * 16;
              if constexpr (EPI == kLbF32) {
                float* out = reinterpret_cast<float*>(args.out) + orow * args.N + n0;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  *reinterpret_cast<float4*>(out + 4 * q) =
                      make_float4(__fmul_rn(__uint_as_float(v[4 * q]), 16.0f),
                                  __fmul_rn(__uint_as_float(v[4 * q + 1]), 16.0f),
                                  __fmul_rn(__uint_as_float(v[4 * q + 2]), 16.0f),
                                  __fmul_rn(__uint_as_float(v[4 * q + 3]), 16.0f));
              } else {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float y0 = __fmul_rn(__fmul_rn(__uint_as_float(v[2 * i]), 16.0f),
                                             __fmul_rn(sx, sc[2 * i]));
                  const float y1 = __fmul_rn(__fmul_rn(__uint_as_float(v[2 * i + 1]), 16.0f),
                                             __fmul_rn(sx, sc[2 * i + 1]));
                  const __nv_bfloat162 pr = __floats2bfloat162_rn(y0, y1);
                  w[i] = *reinterpret_cast<const uint32_t*>(&pr);
                }
                uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(args.out) +
                                                      orow * args.N + n0);
                out[0] = make_uint4(w[0], w[1], w[2], w[3]);
                out[1] = make_uint4(w[4], w[5], w[6], w[7]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
        else
          mbar_arrive(&tempty[acc]);
      }
    }
  }

  __syncthreads();
  int never = 0;
  if (*abort_flag) {
    // after a timeout: let every issued copy and MMA land before the shared
    // memory and the TMEM columns are released
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < R; ++s)
        if (issued_mask & (1u << s))
          mbar_wait_limit(&raw_full[s], (issued_parity >> s) & 1u, &never, kErrTimeoutTeardown,
                          100000000ull);
    }
    if (warp == 1 && lane == 0 && leader && mma_issued) {
      if constexpr (PAIR)
        umma_commit_pair(drain, 0x1);
      else
        umma_commit(drain);
      mbar_wait_limit(drain, 0, &never, kErrTimeoutTeardown, 100000000ull);
    }
    __syncthreads();
  }
  if constexpr (PAIR) {
    // neither CTA releases the pair's TMEM or leaves while the other may still
    // signal its barriers or read its shared memory (bounded)
    if (threadIdx.x == 0) {
      mbar_arrive_cluster(mapa_shared(smem_u32(fin), rank ^ 1u));
      mbar_wait_limit(fin, 0, &never, kErrTimeoutTeardown, 1000000000ull);
    }
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, lb::kTmemCols);
    else
      tmem_dealloc(tmem_base, lb::kTmemCols);
  }
}

}  // namespace convrot
