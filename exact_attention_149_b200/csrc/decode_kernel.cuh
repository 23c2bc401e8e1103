// Paged split-KV decode for sm_100a ("FlashAttention 实战指南" §增量解码场景
// flash_attn_with_kvcache: append the new K/V to the cache in place, attend
// in place; cache_seqlens gives each sample's length, block_table pages the
// cache, num_splits splits the KV range; rotary_cos / rotary_sin rotate q and
// the new keys inside the call).
//
//   kv_append_kernel     the Sq new K/V rows -> their page slots (positions
//                        cache_seqlens[b] ..), keys rotated when rotary tables
//                        are given; with rotary, also the rotated queries into
//                        the workspace
//   decode_split_kernel  one CTA per (sequence, kv head, split, column block):
//                        a TMA producer warp streams 64-token K/V chunks of
//                        the split's range through block_table into a shared-
//                        memory ring; four consumer warps each own 16 tokens of
//                        a chunk and keep an online softmax for up to 32 query
//                        columns, a column being one (new token, query head of
//                        the GQA group) pair, so every K/V byte is read from
//                        HBM once per column block.
//   lse_combine_kernel   merges the splits' (O_s, LSE_s) partials.
//
// Decode is bound by HBM bandwidth (about 4 flops per K/V byte), so the dot
// products run on mma.sync (m16n8k16) straight from the swizzled TMA tiles:
//   S^T[16 tokens x 8 columns] = K[16 x 16 d] . Q^T[16 d x 8 columns]
//   O^T[16 d x 8 columns]     += V^T[16 d x 16 tokens] . P^T[16 tokens x 8 columns]
// P^T's fragment is the transpose of S^T's accumulator fragment, done with
// movmatrix.
//
// int8 / int4 caches: the chunks arrive as codes plus one float32 scale per
// (token, kv head) row. At D = 128 each consumer lane builds its mma
// fragments straight from the code tiles in registers (codes become exact
// fp16 by placing them under the exponent bits of 1024 and subtracting the
// bias), with the head dimension permuted per lane so that its loads are
// 16-byte reads; QK then runs in fp16 on queries scaled by a power of two.
// At D = 64 (int8 only) each warp converts its 16 rows into 16-bit tiles in
// its own shared memory and the products above run on them. Either way the K
// scale multiplies the rows of S^T, and the V scale, divided by the largest
// V scale the warp has seen, multiplies P (so the fp16 P keeps 11 bits
// without overflow); that largest scale is folded into the accumulator's
// online rescale.
#pragma once

#include "ptx.cuh"

namespace fa {

enum : int { kDevBadIndex = 2 };

struct DecodeParams {
  const void* q;          // (B, Sq, Hq, D): the caller's q, or the rotated copy
  const void* q_in;       // the caller's q (read by kv_append_kernel)
  void* q_rot;            // (B, Sq, Hq, D) rotated queries (workspace), or null
  const void* k_new;      // (B, Sq, Hkv, D) or null
  const void* v_new;
  void* k_cache;          // (num_pages, page_size, Hkv, D)
  void* v_cache;
  const int* block_table; // (B, max_pages); null: contiguous cache, page b = sequence b
  const int* cache_seqlens;
  const float* rot_cos;   // (rot_rows, rot_dim / 2) fp32, or null
  const float* rot_sin;
  void* out;              // (B, Sq, Hq, D)
  float* lse;             // (B, Hq, Sq)
  float* part_o;          // (splits, B, Sq, Hq, D) fp32, used when splits > 1
  float* part_lse;        // (splits, B, Sq, Hq)
  int B, Sq, Hq, Hkv, D, group;
  int n_cols;             // Sq * group query columns per (sequence, kv head)
  int col_blocks;         // column blocks of 8 * kNT columns
  int page_size, max_pages, num_pages;
  int splits;
  int append;             // 1 when k_new/v_new are given
  int rot_rows, rot_dim, rot_inter;
  float scale_log2, softcap, cap_in, cap_out_log2;
  int wl;                 // window left (-1 = unbounded)
  int right;              // visible keys end at position + right (-1 = unbounded; causal = 0)
  const float* alibi;     // ALiBi slopes, nullable: slope of (b, hq) = alibi[b * alibi_bstride + hq]
  int alibi_bstride;
  // int8 cache: k_cache / v_cache hold codes, these the per-row scales,
  // (num_pages, Hkv, page_size) fp32; null for a 16-bit cache
  float* k_scale;
  float* v_scale;
};

// Keys visible to the query at position `qpos` of a sequence of Lk keys:
// [key_lo, key_hi). Bottom-right alignment: the last query sits at Lk - 1.
__device__ __forceinline__ int key_lo(const DecodeParams& p, int qpos) {
  return p.wl >= 0 ? max(0, qpos - p.wl) : 0;
}
__device__ __forceinline__ int key_hi(const DecodeParams& p, int qpos, int Lk) {
  return p.right >= 0 ? min(Lk, qpos + p.right + 1) : Lk;
}

// ---------------------------------------------------------------------------
// append (+ rotary)
// ---------------------------------------------------------------------------
template <bool kBF16>
__device__ __forceinline__ void unpack8(const uint4& r, float (&x)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = unpack2<kBF16>(w[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
template <bool kBF16>
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  return make_uint4(pack2<kBF16>(x[0], x[1]), pack2<kBF16>(x[2], x[3]), pack2<kBF16>(x[4], x[5]),
                    pack2<kBF16>(x[6], x[7]));
}

// Elements d0 .. d0+7 of one head row after the rotary rotation at the angle
// row (cs, sn) (null: no rotation). A pair (a, b) becomes
// (a cos - b sin, a sin + b cos); pairs are (i, i + rd/2), or (2i, 2i + 1)
// when interleaved; dimensions from rd on pass through. rd is a multiple of
// 16, so a group of 8 never straddles rd or rd/2.
template <bool kBF16>
__device__ __forceinline__ uint4 rotate8(const uint16_t* row, int d0, const float* cs,
                                         const float* sn, const DecodeParams& p) {
  const uint4 raw = *reinterpret_cast<const uint4*>(row + d0);
  if (cs == nullptr || d0 >= p.rot_dim) return raw;
  float x[8], y[8];
  unpack8<kBF16>(raw, x);
  if (p.rot_inter) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float c = cs[(d0 >> 1) + j], s = sn[(d0 >> 1) + j];
      y[2 * j] = x[2 * j] * c - x[2 * j + 1] * s;
      y[2 * j + 1] = x[2 * j] * s + x[2 * j + 1] * c;
    }
  } else {
    const int half = p.rot_dim >> 1;
    const bool first = d0 < half;
    const int i0 = first ? d0 : d0 - half;
    float xp[8];
    unpack8<kBF16>(*reinterpret_cast<const uint4*>(row + (first ? d0 + half : d0 - half)), xp);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float c = cs[i0 + j], s = sn[i0 + j];
      y[j] = first ? x[j] * c - xp[j] * s : xp[j] * s + x[j] * c;
    }
  }
  return pack8<kBF16>(y);
}

// Symmetric quantisation of one head row of D values held by 16 lanes (8
// consecutive values each; lanes at or past D / 8 hold zeros): scale = max|x|
// / qmax, code = round-half-even(x / scale), both in fp32 with IEEE
// division; a zero row has scale 0 and codes 0. qmax is 127 (kQ = 8) or 7
// (kQ = 4). Returns the lane's 8 codes: int8, little-endian in two words; int4,
// biased by 8, two per byte (even d in the low nibble) in .x. *scale gets
// the row's scale.
template <int kQ>
__device__ __forceinline__ uint2 quantize_row(const float (&x)[8], float* scale) {
  constexpr int kMax = kQ == 8 ? 127 : 7;
  float am = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(x[j]));
#pragma unroll
  for (int off = 1; off < 16; off <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
  const float sc = __fdiv_rn(am, static_cast<float>(kMax));
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    int c = sc > 0.f ? __float2int_rn(__fdiv_rn(x[j], sc)) : 0;
    c = max(-kMax, min(kMax, c));
    if constexpr (kQ == 8)
      w[j >> 2] |= (static_cast<uint32_t>(c) & 0xffu) << (8 * (j & 3));
    else
      w[0] |= static_cast<uint32_t>(c + 8) << (4 * j);
  }
  *scale = sc;
  return make_uint2(w[0], w[1]);
}

// grid B * Sq (one block per new token), block 128: 16 bytes per thread-step.
// kQuant: the new rows are quantised into an int8 / int4 cache (keys after the rotary
// rotation and the rounding to the 16-bit type, as the 16-bit cache stores
// them); each warp takes heads warp, warp + 4, ..., lanes 0-15 the key row and
// lanes 16-31 the value row.
template <bool kBF16, int kQ>
__global__ void kv_append_kernel(const DecodeParams p) {
  constexpr bool kQuant = kQ != 0;
  const int b = blockIdx.x / p.Sq, t = blockIdx.x % p.Sq;
  const int L = p.cache_seqlens[b];
  const int Lk = L + (p.append ? p.Sq : 0);
  const int pos = Lk - p.Sq + t;  // position of query t and of new key t
  const float* cs = nullptr;
  const float* sn = nullptr;
  if (p.rot_dim > 0) {
    if (L < 0 || pos < 0 || pos >= p.rot_rows) {
      if (threadIdx.x == 0) atomicExch(&g_device_status, kDevBadIndex);
    } else {
      cs = p.rot_cos + static_cast<size_t>(pos) * (p.rot_dim >> 1);
      sn = p.rot_sin + static_cast<size_t>(pos) * (p.rot_dim >> 1);
    }
    const int groups = p.D >> 3;
    const size_t base = (static_cast<size_t>(b) * p.Sq + t) * p.Hq * p.D;
    const uint16_t* src = static_cast<const uint16_t*>(p.q_in) + base;
    uint16_t* dst = static_cast<uint16_t*>(p.q_rot) + base;
    for (int i = threadIdx.x; i < p.Hq * groups; i += blockDim.x) {
      const int h = i / groups, d0 = (i % groups) * 8;
      *reinterpret_cast<uint4*>(dst + h * p.D + d0) = rotate8<kBF16>(src + h * p.D, d0, cs, sn, p);
    }
  }
  if (!p.append) return;
  if (L < 0 || Lk > p.max_pages * p.page_size) {
    if (threadIdx.x == 0) atomicExch(&g_device_status, kDevBadIndex);
    return;
  }
  const int page =
      p.block_table ? p.block_table[static_cast<size_t>(b) * p.max_pages + pos / p.page_size] : b;
  if (page < 0 || page >= p.num_pages) {
    if (threadIdx.x == 0) atomicExch(&g_device_status, kDevBadIndex);
    return;
  }
  const int groups = p.D >> 3;
  const size_t dst = (static_cast<size_t>(page) * p.page_size + (pos % p.page_size)) * p.Hkv * p.D;
  const size_t src = (static_cast<size_t>(b) * p.Sq + t) * p.Hkv * p.D;
  const uint16_t* kn = static_cast<const uint16_t*>(p.k_new) + src;
  const uint16_t* vn = static_cast<const uint16_t*>(p.v_new) + src;
  if constexpr (kQuant) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, li = lane & 15;
    const bool act = li < groups;
    for (int h = warp; h < p.Hkv; h += blockDim.x >> 5) {
      float x[8];
      if (act) {
        const uint4 raw = half == 0 ? rotate8<kBF16>(kn + h * p.D, li * 8, cs, sn, p)
                                    : *reinterpret_cast<const uint4*>(vn + h * p.D + li * 8);
        unpack8<kBF16>(raw, x);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = 0.f;
      }
      float sc;
      const uint2 codes = quantize_row<kQ>(x, &sc);
      uint8_t* cache = static_cast<uint8_t*>(half == 0 ? p.k_cache : p.v_cache);
      if (act) {
        if constexpr (kQ == 8)
          *reinterpret_cast<uint2*>(cache + dst + h * p.D + li * 8) = codes;
        else  // two codes per byte
          *reinterpret_cast<uint32_t*>(cache + (dst + h * p.D + li * 8) / 2) = codes.x;
      }
      if (li == 0) {
        float* scales = half == 0 ? p.k_scale : p.v_scale;
        scales[(static_cast<size_t>(page) * p.Hkv + h) * p.page_size + pos % p.page_size] = sc;
      }
    }
    return;
  }
  uint16_t* kc = static_cast<uint16_t*>(p.k_cache) + dst;
  uint16_t* vc = static_cast<uint16_t*>(p.v_cache) + dst;
  for (int i = threadIdx.x; i < p.Hkv * groups; i += blockDim.x) {
    const int h = i / groups, d0 = (i % groups) * 8;
    const int e = h * p.D + d0;
    *reinterpret_cast<uint4*>(kc + e) = rotate8<kBF16>(kn + h * p.D, d0, cs, sn, p);
    *reinterpret_cast<uint4*>(vc + e) = *reinterpret_cast<const uint4*>(vn + e);
  }
}

// A 16-bit cache (rows, Hkv, D), rows = num_pages * page_size, into int8
// codes of the same shape (or int4 codes, two per byte: (rows, Hkv, D / 2))
// and scales (num_pages, Hkv, page_size): one (row, head) unit per 16-lane
// half-warp, eight units per 128-thread block.
template <bool kBF16, int kQ>
__global__ void kv_quantize_kernel(const uint16_t* src, uint8_t* codes, float* scales, long long units,
                                   int Hkv, int D, int page_size) {
  const int li = threadIdx.x & 15;
  const long long u = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 4);
  const bool act = u < units && li < (D >> 3);
  float x[8];
  if (act) {
    unpack8<kBF16>(*reinterpret_cast<const uint4*>(src + u * D + li * 8), x);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = 0.f;
  }
  float sc;
  const uint2 c = quantize_row<kQ>(x, &sc);
  if (act) {
    if constexpr (kQ == 8)
      *reinterpret_cast<uint2*>(codes + u * D + li * 8) = c;
    else
      *reinterpret_cast<uint32_t*>(codes + (u * D + li * 8) / 2) = c.x;
  }
  if (u < units && li == 0) {
    const long long row = u / Hkv;
    const int h = static_cast<int>(u % Hkv);
    scales[((row / page_size) * Hkv + h) * page_size + row % page_size] = sc;
  }
}

// Two biased codes (code + 128, bytes 0, 1 of w, or bytes 2, 3 with hi) ->
// their exact fp16 pair: 0x64 above a biased byte is the fp16 value 1024 +
// code + 128, and subtracting 1152 leaves the code.
__device__ __forceinline__ uint32_t i8pair_to_f16(uint32_t w, bool hi) {
  const uint32_t h = __byte_perm(w, 0x64646464u, hi ? 0x4342u : 0x4140u);
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h),
                            __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// The biased int4 codes (code + 8) in bits 0-3 and 16-19 of w -> their exact
// fp16 pair: 0x64 above the nibble is the fp16 value 1024 + code + 8, and
// subtracting 1032 leaves the code.
__device__ __forceinline__ uint32_t i4pair_to_f16(uint32_t w) {
  const uint32_t h = (w & 0x000F000Fu) | 0x64006400u;
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h),
                            __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// The same for the codes in bits 4-7 and 20-23, left in place: 0x64 above
// them is 1024 + 16 (code + 8), and subtracting 1152 leaves 16 * code (exact;
// the caller undoes the factor 16 elsewhere, saving the shift).
__device__ __forceinline__ uint32_t i4pair_hi_to_f16x16(uint32_t w) {
  const uint32_t h = (w & 0x00F000F0u) | 0x64006400u;
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h),
                            __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// 16 int8 codes -> 16 exact 16-bit values (two uint4 of 8), without the
// special-function unit. bf16: each biased byte (code + 128) becomes the low
// mantissa byte of 2^23, so the fp32 value is 2^23 + code + 128; subtracting
// 2^23 + 128 leaves the code, whose upper 16 bits are its exact bf16. fp16:
// 0x64 above a biased byte is the fp16 value 1024 + code + 128; subtracting
// 1152 leaves the code.
template <bool kBF16>
__device__ __forceinline__ void i8x16_to_16bit(const uint4& a, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t u = w[i] ^ 0x80808080u;
    if constexpr (kBF16) {
      const float2 bias = make_float2(-8388736.f, -8388736.f);
      const float2 f01 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)),
                                                __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541))),
                                    bias);
      const float2 f23 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)),
                                                __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543))),
                                    bias);
      o[2 * i] = __byte_perm(__float_as_uint(f01.x), __float_as_uint(f01.y), 0x7632);
      o[2 * i + 1] = __byte_perm(__float_as_uint(f23.x), __float_as_uint(f23.y), 0x7632);
    } else {
      const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152
      const uint32_t h01 = __byte_perm(u, 0x64646464u, 0x4140);
      const uint32_t h23 = __byte_perm(u, 0x64646464u, 0x4342);
      const __half2 r01 = __hsub2(*reinterpret_cast<const __half2*>(&h01), bias);
      const __half2 r23 = __hsub2(*reinterpret_cast<const __half2*>(&h23), bias);
      o[2 * i] = *reinterpret_cast<const uint32_t*>(&r01);
      o[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&r23);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// 32 int4 codes (16 bytes; byte i holds code 2i + 8 in its low nibble and
// code 2i + 1 + 8 in its high one) -> 32 exact 16-bit values in d order. For
// each byte one permute puts it in bytes 0 and 2, one AND/OR against
// 0x64006400 makes the fp16 pair (1024 + low, 1024 + 16 high), and one
// packed FMA by (1, 1/16) minus (1032, 72) leaves the two codes (exact).
// bf16 takes the exact fp16 values through float.
template <bool kBF16>
__device__ __forceinline__ void i4x32_to_16bit(const uint4& a, uint4 (&o)[4]) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  const __half2 mul = __halves2half2(__float2half_rn(1.f), __float2half_rn(0.0625f));
  const __half2 sub = __halves2half2(__float2half_rn(-1032.f), __float2half_rn(-72.f));
  uint32_t r[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t t = __byte_perm(w[i], 0u, static_cast<uint32_t>(k | (4 << 4) | (k << 8) | (4 << 12)));
      const uint32_t h = (t & 0x00F0000Fu) | 0x64006400u;
      const __half2 c = __hfma2(*reinterpret_cast<const __half2*>(&h), mul, sub);
      if constexpr (kBF16) {
        const float2 f = __half22float2(c);
        r[4 * i + k] = pack2<true>(f.x, f.y);
      } else {
        r[4 * i + k] = *reinterpret_cast<const uint32_t*>(&c);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) o[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
}

// ---------------------------------------------------------------------------
// warp-level tensor-core helpers (legacy mma.sync path)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
template <bool kBF16>
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (kBF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// int4 slices: the token (0..15 within a warp's 16) that fragment row / k
// index m stands for, m ^ ((m >> 1) & 1): rows m = r and r + 8 of the K
// fragment and k = 2j + {0, 1, 8, 9} of the V fragment then fall, under the
// 64-byte swizzle of the 64-byte int4 rows, on distinct banks. S^T row m and
// P^T column m are the same token, so only the addressing and the token
// positions change.
__device__ __forceinline__ int i4_token(int m) { return m ^ ((m >> 1) & 1); }

// address of the 16-byte group `g` (0..7 within a 128-byte row) of row `r`
// of a TMA tile written with the 128-byte swizzle (tile base 1024-aligned)
__device__ __forceinline__ uint32_t sw128(uint32_t base, int r, int g) {
  return base + r * 128 + ((g ^ (r & 7)) << 4);
}

// kQuant: the ring holds int8 / int4 chunks (K codes, V codes, then the 64 K and 64 V
// scales). D = 128: int8 code tiles arrive with the 128-byte swizzle, int4
// tiles (64-byte rows) with the 64-byte swizzle, and the consumers build their
// fragments from them in registers. D = 64 (int8 64-byte rows, int4 32-byte
// rows): unswizzled tiles, and each consumer warp converts its 16 rows into
// 16-bit tiles in its own scratch (K then V, 16 rows x 128 B in the 128-byte
// swizzle of the TMA tiles) before the tensor-core steps.
template <int kD, int kQ = 0>
struct DecShape {
  static constexpr bool kQuant = kQ != 0;           // an int8 (kQ = 8) or int4 (kQ = 4) cache
  static constexpr int kRowBytes = kD * (kQuant ? kQ : 16) / 8;  // one cached row of one head
  static constexpr int kTok = 64;                      // tokens per chunk
  static constexpr int kChunks = kD / 64;              // 128-byte column chunks
  static constexpr int kBoxBytes = kTok * 128;         // 64 rows x 128 B
  static constexpr int kKVBytes = kQuant ? kTok * kRowBytes : kChunks * kBoxBytes;  // K or V of one chunk
  static constexpr int kScaleOffset = 2 * kKVBytes;    // int8: 64 K scales, 64 V scales
  // bytes the producer loads into a stage (the full barrier's transaction
  // count); int8 stages are padded to 1 KB, which the 128-byte-swizzled TMA
  // tiles need, so the stage stride can exceed the loaded bytes
  static constexpr int kLoadBytes = 2 * kKVBytes + (kQuant ? 2 * kTok * 4 : 0);
  static constexpr int kStageBytes = kQuant ? (kLoadBytes + 1023) / 1024 * 1024 : kLoadBytes;
  // 2 (16-bit) or 3 CTAs per SM; int4 keeps 8 stages so that the cross-warp
  // reduction scratch, which aliases the ring, fits
  // (16-bit D = 256: 64 KB stages, three of them, one CTA per SM)
  static constexpr int kStages =
      kQuant ? (kQ == 4 ? 8 : (kD == 128 ? 4 : 6)) : (kD == 256 ? 3 : (kD == 128 ? 3 : 6));
  // int8 with D = 128 builds the tensor-core fragments straight from the
  // swizzled int8 tiles in registers; D = 64 converts through a scratch
  static constexpr bool kDirect = kQuant && kD == 128;
  static constexpr int kScrHalfBytes = kChunks * 16 * 128;   // 16 rows of K (or V), 16-bit
  static constexpr int kScrOffset = kStages * kStageBytes;
  static constexpr int kScrBytes = (kQuant && !kDirect) ? 4 * 2 * kScrHalfBytes : 0;
  static constexpr int kBarOffset = kScrOffset + kScrBytes;
  // cross-warp reduction scratch aliases the stage ring (and the int8
  // scratch): it is written only after every issued chunk has been consumed
  static constexpr int kRedOffset = 0;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;
  static constexpr int kThreads = 160;                 // 4 consumer warps + 1 producer
  static_assert(kScrOffset % 1024 == 0 && kStageBytes % 128 == 0, "scratch and stage alignment");
  static_assert(kStages <= 8, "more ring slots than the barrier block holds");
};

struct DecBars {
  uint64_t full[8];
  uint64_t empty[8];
  int abort;
};

__device__ __forceinline__ float dec_logit(float s, const DecodeParams& p) {
  if (p.softcap > 0.f) return p.cap_out_log2 * tanh_fast(s * p.cap_in);
  return s * p.scale_log2;
}

// kNT: number of 8-wide column tiles per CTA (a column block holds 8 * kNT
// columns; column n is new token n / group, query head kvh * group + n % group)
template <int kD, bool kBF16, int kNT, int kQ>
__global__ void __launch_bounds__(160)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using Sh = DecShape<kD, kQ>;
  constexpr bool kQuant = Sh::kQuant;
  constexpr bool kQ4 = kQ == 4;
  static_assert(sizeof(DecBars) <= 256, "barrier block exceeds its reservation");
  static_assert((8 * 8 * kNT + 4 * 8 * kNT * kD) * 4 <= Sh::kBarOffset, "reduction scratch exceeds the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DecBars* bars = reinterpret_cast<DecBars*>(smem + Sh::kBarOffset);
  float* red = reinterpret_cast<float*>(smem + Sh::kRedOffset);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kH = 8 * kNT;
  // work item: column block fastest (the blocks of one split read the same
  // K/V, so they run together and share it through L2), then split, kv head,
  // sequence
  const int cb = blockIdx.x % p.col_blocks;
  const int split = (blockIdx.x / p.col_blocks) % p.splits;
  const int kvh = (blockIdx.x / (p.col_blocks * p.splits)) % p.Hkv;
  const int b = blockIdx.x / (p.col_blocks * p.splits * p.Hkv);
  const int n0 = cb * kH;                        // first column of the block
  const int n_here = min(kH, p.n_cols - n0);     // real columns in the block

  const int L = p.cache_seqlens[b];
  const int Lk = L + (p.append ? p.Sq : 0);      // keys after the append
  const int qbase = Lk - p.Sq;                   // position of new token 0
  // union [lo, hi) and intersection [lo_in, hi_in) of the block's columns'
  // key ranges: both bounds grow with the token index
  const int t_first_col = n0 / p.group, t_last_col = (n0 + n_here - 1) / p.group;
  const int lo = key_lo(p, qbase + t_first_col);
  const int hi = key_hi(p, qbase + t_last_col, Lk);  // exclusive
  const int lo_in = key_lo(p, qbase + t_last_col);
  const int hi_in = key_hi(p, qbase + t_first_col, Lk);
  const int t_first = lo / Sh::kTok;
  const int t_all = hi > lo ? (hi - 1) / Sh::kTok + 1 - t_first : 0;
  const int per = (t_all + p.splits - 1) / p.splits;
  const int t_begin = t_first + split * per;
  const int t_end = min(t_first + t_all, t_begin + per);
  const int n_t = max(0, t_end - t_begin);
  const bool bad_len = (L < 0) || (Lk > p.max_pages * p.page_size);

  if (threadIdx.x == 0) {
    for (int i = 0; i < Sh::kStages; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 4);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &bars->abort;
  const int n_iter = bad_len ? 0 : n_t;
  if (bad_len && threadIdx.x == 0) atomicExch(&g_device_status, kDevBadIndex);

  if (warp == 4) {
    // ======================= producer =======================
    if (elect_one()) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int* bt = p.block_table ? p.block_table + static_cast<size_t>(b) * p.max_pages : nullptr;
      int i = 0;
      for (; i < n_iter; ++i) {
        const int slot = i % Sh::kStages;
        const uint32_t ph = static_cast<uint32_t>(i / Sh::kStages) & 1u;
        bool ok = mbar_try_wait(&bars->empty[slot], ph ^ 1u);
        if (!ok) {
          const uint64_t t0 = globaltimer_ns();
          for (uint32_t it = 1; !ok; ++it) {
            ok = mbar_try_wait(&bars->empty[slot], ph ^ 1u);
            if (!ok && (it & 63u) == 0u &&
                (*abort || globaltimer_ns() - t0 > kWaitTimeoutNs)) {
              atomicExch(&g_device_status, kDevTimeout);
              *abort = 1;
              break;
            }
          }
        }
        if (!ok) break;
        const int pos = (t_begin + i) * Sh::kTok;
        int page = bt ? bt[pos / p.page_size] : b;
        if (page < 0 || page >= p.num_pages) {
          atomicExch(&g_device_status, kDevBadIndex);
          page = 0;  // stay in bounds; the result is flagged as invalid
        }
        const int row = page * p.page_size + (pos % p.page_size);
        mbar_arrive_expect_tx(&bars->full[slot], Sh::kLoadBytes);
        uint8_t* dst = smem + slot * Sh::kStageBytes;
        if constexpr (kQuant) {
          // one box of 64 rows x kD bytes each, then the chunk's scales: 64
          // contiguous floats of (page, kvh) (page_size is a multiple of 64)
          tma_load_3d(&tm_k, &bars->full[slot], dst, 0, kvh, row);
          tma_load_3d(&tm_v, &bars->full[slot], dst + Sh::kKVBytes, 0, kvh, row);
          const size_t so = (static_cast<size_t>(page) * p.Hkv + kvh) * p.page_size + pos % p.page_size;
          bulk_load(dst + Sh::kScaleOffset, p.k_scale + so, Sh::kTok * 4, &bars->full[slot]);
          bulk_load(dst + Sh::kScaleOffset + Sh::kTok * 4, p.v_scale + so, Sh::kTok * 4, &bars->full[slot]);
        } else {
          for (int c = 0; c < Sh::kChunks; ++c) {
            tma_load_3d(&tm_k, &bars->full[slot], dst + c * Sh::kBoxBytes, c * 64, kvh, row);
            tma_load_3d(&tm_v, &bars->full[slot], dst + Sh::kKVBytes + c * Sh::kBoxBytes, c * 64, kvh,
                        row);
          }
        }
      }
      // drain the loads still in flight
      for (int f = max(0, i - Sh::kStages); f < i; ++f)
        mbar_wait(&bars->full[f % Sh::kStages], static_cast<uint32_t>(f / Sh::kStages) & 1u);
    }
    __syncwarp();
    __syncthreads();
    return;
  }

  // ======================= consumers (warps 0..3) =======================
  // Q^T fragments: B[k = d][n = column], n = lane / 4 within each 8-column tile
  uint32_t qf[kNT][kD / 16][2];
  // int8, D = 128: the contraction index is permuted so that lane j = lane % 4
  // owns d in [32 j, 32 j + 32): K-step kk, fragment k = 2j, 2j+1 <-> d =
  // 32j + 4kk + {0, 1} and k = 2j+8, 2j+9 <-> d = 32j + 4kk + {2, 3}. The
  // queries enter as fp16, each column scaled by an exact power of two 2^-e
  // (its largest |q| lands in [2^14, 2^15)); qsc holds 2^e of this lane's two
  // accumulator columns 2j, 2j+1.
  float qsc[kNT][2];
  if constexpr (Sh::kDirect) {
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      const int n = n0 + nt * 8 + (lane >> 2);
      const bool real = n < p.n_cols;
      const int t = real ? n / p.group : 0, hl = real ? n % p.group : 0;
      const uint16_t* row = static_cast<const uint16_t*>(p.q) +
                            ((static_cast<size_t>(b) * p.Sq + t) * p.Hq + kvh * p.group + hl) * kD +
                            32 * (lane & 3);
      float v[32];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint2 w = real ? *reinterpret_cast<const uint2*>(row + 4 * kk) : make_uint2(0u, 0u);
        const float2 f0 = unpack2<kBF16>(w.x), f1 = unpack2<kBF16>(w.y);
        v[4 * kk] = f0.x;
        v[4 * kk + 1] = f0.y;
        v[4 * kk + 2] = f1.x;
        v[4 * kk + 3] = f1.y;
      }
      float am = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      // e >= -100 keeps 2^-e finite when every |q| of the column is
      // subnormal (such a column then scales to tiny fp16 values: its scores
      // are 0 to within float32 anyway)
      const int e = am > 0.f ? max(ilogbf(am) - 14, -100) : 0;
      const float down = ldexpf(1.f, -e), up = ldexpf(1.f, e);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if constexpr (kQ4) {
          // int4: K-step kk pairs nibbles (i, i + 4) and (i + 1, i + 5) of
          // word kk / 2, i = 2 (kk % 2): d = 32j + 8 (kk / 2) + i + {0, 4}
          // and + {1, 5}. The K values of the second pair arrive as 16 x
          // code (i4pair_hi_to_f16x16), so their queries carry 1 / 16.
          const int i0 = 8 * (kk >> 1) + 2 * (kk & 1);
          const float down16 = down * 0.0625f;
          qf[nt][kk][0] = pack2<false>(v[i0] * down, v[i0 + 4] * down);
          qf[nt][kk][1] = pack2<false>(v[i0 + 1] * down16, v[i0 + 5] * down16);
        } else {
          qf[nt][kk][0] = pack2<false>(v[4 * kk] * down, v[4 * kk + 1] * down);
          qf[nt][kk][1] = pack2<false>(v[4 * kk + 2] * down, v[4 * kk + 3] * down);
        }
      }
      qsc[nt][0] = __shfl_sync(0xffffffffu, up, 8 * (lane & 3));
      qsc[nt][1] = __shfl_sync(0xffffffffu, up, 8 * (lane & 3) + 4);
    }
  } else {
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      const int n = n0 + nt * 8 + (lane >> 2);
      const bool real = n < p.n_cols;
      const int t = real ? n / p.group : 0, hl = real ? n % p.group : 0;
      const uint16_t* row = static_cast<const uint16_t*>(p.q) +
                            ((static_cast<size_t>(b) * p.Sq + t) * p.Hq + kvh * p.group + hl) * kD;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const int d = kk * 16 + 2 * (lane & 3);
        qf[nt][kk][0] = real ? *reinterpret_cast<const uint32_t*>(row + d) : 0u;
        qf[nt][kk][1] = real ? *reinterpret_cast<const uint32_t*>(row + d + 8) : 0u;
      }
      qsc[nt][0] = qsc[nt][1] = 1.f;
    }
  }
  // ALiBi: slope (exp2 domain) and query position of this lane's columns
  const bool alibi = p.alibi != nullptr;
  float asl[kNT][2], aqp[kNT][2];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = min(n0 + nt * 8 + 2 * (lane & 3) + j, p.n_cols - 1);
      const int hq = kvh * p.group + n % p.group;
      asl[nt][j] = alibi ? p.alibi[static_cast<size_t>(b) * p.alibi_bstride + hq] * 1.4426950408889634f : 0.f;
      aqp[nt][j] = static_cast<float>(qbase + n / p.group);
    }
  }
  // running state per (column tile, column pair): columns nt*8 + 2*(lane&3) + {0,1}
  float m_run[kNT][2], l_part[kNT][2];
  // int8: the PV product runs in fp16 on P * (V row scale / vC), vC the
  // largest V scale this warp has seen, so every factor is <= 1 and keeps
  // fp16's 11-bit precision; acc holds O / vC (vC only grows, and the change
  // is folded into the online-softmax rescale of acc)
  float vC = 1.17549435e-38f;
  float vCinv = 1.f / 1.17549435e-38f;
  float acc[kNT][kD / 16][4];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_part[nt][0] = l_part[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt) acc[nt][mt][0] = acc[nt][mt][1] = acc[nt][mt][2] = acc[nt][mt][3] = 0.f;
  }
  const uint32_t sbase = smem_u32(smem);
  bool ok = true;
  for (int i = 0; i < n_iter; ++i) {
    const int slot = i % Sh::kStages;
    // bounded wait on the chunk
    {
      const uint32_t ph = static_cast<uint32_t>(i / Sh::kStages) & 1u;
      if (!mbar_try_wait(&bars->full[slot], ph)) {
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 1;; ++it) {
          if (mbar_try_wait(&bars->full[slot], ph)) break;
          if ((it & 63u) == 0u && (*abort || globaltimer_ns() - t0 > kWaitTimeoutNs)) {
            atomicExch(&g_device_status, kDevTimeout);
            *abort = 1;
            ok = false;
            break;
          }
        }
      }
      if (!ok) break;
    }
    const int tok0 = warp * 16;  // this warp's 16 tokens of the chunk
    // 16-bit tiles the tensor-core steps read: the TMA chunk itself, or (int8)
    // this warp's converted rows, addressed by the row within the tile
    uint32_t kbase = sbase + slot * Sh::kStageBytes;
    uint32_t vbase = kbase + Sh::kKVBytes;
    constexpr int kTileStride = kQuant ? 16 * 128 : Sh::kBoxBytes;  // per 64-column chunk
    const int trow0 = kQuant ? tok0 : 0;                            // tile row = token - trow0
    float ksc0 = 1.f, ksc1 = 1.f, vsc0 = 1.f, vsc1 = 1.f;
    // direct int8 path: this lane's code words. K: rows tok0 + r and
    // tok0 + r + 8 (r = lane / 4), bytes d = 32j .. 32j + 31 (j = lane % 4);
    // V: tokens tok0 + 2j + {0, 1, 8, 9}, bytes d = 16r .. 16r + 15. Rows are
    // 128 bytes with the 16-byte group g stored at g ^ (row & 7).
    uint32_t kw[2][8], vw[4][4];
    if constexpr (kQ4 && Sh::kDirect) {
      // int4 rows are 64 bytes, written by TMA with the 64-byte swizzle (the
      // 16-byte group g of row t at g ^ ((t >> 1) & 3)). Fragment row / k
      // index m of the warp's 16 tokens is token tok0 + i4_token(m), so that
      // both reads below are free of bank conflicts. K: this lane's 16 bytes
      // (d = 32j .. 32j + 31) of tokens i4_token(r), i4_token(r + 8); V, its
      // 8 bytes (d = 16r .. 16r + 15) of tokens i4_token(2j + {0, 1, 8, 9}).
      // Codes stay biased by 8.
      const int r = lane >> 2, j = lane & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int tk = tok0 + i4_token(r + 8 * h);
        const uint4 w = *reinterpret_cast<const uint4*>(smem + (kbase - sbase) + tk * 64 +
                                                        ((j ^ ((tk >> 1) & 3)) << 4));
        kw[h][0] = w.x;
        kw[h][1] = w.y;
        kw[h][2] = w.z;
        kw[h][3] = w.w;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int tk = tok0 + i4_token(2 * j + (u & 1) + 8 * (u >> 1));
        const uint2 w = *reinterpret_cast<const uint2*>(smem + (vbase - sbase) + tk * 64 +
                                                        (((r >> 1) ^ ((tk >> 1) & 3)) << 4) + 8 * (r & 1));
        vw[u][0] = w.x;
        vw[u][1] = w.y;
      }
      const float* sc = reinterpret_cast<const float*>(smem + slot * Sh::kStageBytes + Sh::kScaleOffset);
      const int tr = tok0 + i4_token(r);
      ksc0 = sc[tr];
      ksc1 = sc[tr + 8];
      vsc0 = sc[Sh::kTok + tr];
      vsc1 = sc[Sh::kTok + tr + 8];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[slot]);
    } else if constexpr (Sh::kDirect) {
      const int r = lane >> 2, j = lane & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t rb = kbase + (tok0 + r + 8 * h) * 128;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(smem + (rb - sbase) + (((2 * j + c) ^ r) << 4));
          kw[h][4 * c] = w.x ^ 0x80808080u;
          kw[h][4 * c + 1] = w.y ^ 0x80808080u;
          kw[h][4 * c + 2] = w.z ^ 0x80808080u;
          kw[h][4 * c + 3] = w.w ^ 0x80808080u;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int tk = tok0 + 2 * j + (u & 1) + 8 * (u >> 1);
        const uint4 w = *reinterpret_cast<const uint4*>(smem + (vbase - sbase) + tk * 128 + ((r ^ (tk & 7)) << 4));
        vw[u][0] = w.x ^ 0x80808080u;
        vw[u][1] = w.y ^ 0x80808080u;
        vw[u][2] = w.z ^ 0x80808080u;
        vw[u][3] = w.w ^ 0x80808080u;
      }
      const float* sc = reinterpret_cast<const float*>(smem + slot * Sh::kStageBytes + Sh::kScaleOffset);
      ksc0 = sc[tok0 + r];
      ksc1 = sc[tok0 + r + 8];
      vsc0 = sc[Sh::kTok + tok0 + r];
      vsc1 = sc[Sh::kTok + tok0 + r + 8];
      __syncwarp();
      // everything this warp needs from the slot is in registers
      if (lane == 0) mbar_arrive(&bars->empty[slot]);
    } else if constexpr (kQ4) {
      // int4 at D = 64: 32-byte rows, unswizzled; lane = (row r, half u)
      // converts values 32u .. 32u + 31 of its row into the 16-bit groups
      // 4u .. 4u + 3 of the swizzled 128-byte scratch row
      static_assert(kD == 64, "the int4 scratch path is written for D = 64");
      const uint8_t* kq = smem + slot * Sh::kStageBytes + tok0 * Sh::kRowBytes;
      const uint8_t* vq = kq + Sh::kKVBytes;
      uint8_t* ks = smem + Sh::kScrOffset + warp * 2 * Sh::kScrHalfBytes;
      uint8_t* vs = ks + Sh::kScrHalfBytes;
      {
        const int r = lane >> 1, u = lane & 1;
        uint4 o[4];
        i4x32_to_16bit<kBF16>(*reinterpret_cast<const uint4*>(kq + r * Sh::kRowBytes + u * 16), o);
#pragma unroll
        for (int g = 0; g < 4; ++g)
          *reinterpret_cast<uint4*>(ks + r * 128 + (((4 * u + g) ^ (r & 7)) << 4)) = o[g];
        i4x32_to_16bit<false>(*reinterpret_cast<const uint4*>(vq + r * Sh::kRowBytes + u * 16), o);
#pragma unroll
        for (int g = 0; g < 4; ++g)
          *reinterpret_cast<uint4*>(vs + r * 128 + (((4 * u + g) ^ (r & 7)) << 4)) = o[g];
      }
      // the row scales of this lane's accumulator rows (tokens lane / 4, + 8)
      const float* sc = reinterpret_cast<const float*>(smem + slot * Sh::kStageBytes + Sh::kScaleOffset);
      ksc0 = sc[tok0 + (lane >> 2)];
      ksc1 = sc[tok0 + (lane >> 2) + 8];
      vsc0 = sc[Sh::kTok + tok0 + (lane >> 2)];
      vsc1 = sc[Sh::kTok + tok0 + (lane >> 2) + 8];
      __syncwarp();
      // everything this warp needs from the slot is copied out
      if (lane == 0) mbar_arrive(&bars->empty[slot]);
      kbase = smem_u32(ks);
      vbase = smem_u32(vs);
    } else if constexpr (kQuant) {
      const uint8_t* kq = smem + slot * Sh::kStageBytes + tok0 * kD;
      const uint8_t* vq = kq + Sh::kKVBytes;
      uint8_t* ks = smem + Sh::kScrOffset + warp * 2 * Sh::kScrHalfBytes;
      uint8_t* vs = ks + Sh::kScrHalfBytes;
      // 16-byte pieces of the 16 rows: piece j = row (j / (kD/16)), values
      // 16u .. 16u+15 (u = j % (kD/16)) -> column chunk u / 4, 16-byte
      // groups 2 (u % 4) and 2 (u % 4) + 1 of the swizzled 128-byte row
#pragma unroll
      for (int j = lane; j < kD; j += 32) {
        const int r = j / (kD / 16), u = j % (kD / 16);
        const int c = u >> 2, g0 = (u & 3) * 2;
        uint4 lo, hi;
        i8x16_to_16bit<kBF16>(*reinterpret_cast<const uint4*>(kq + r * kD + u * 16), lo, hi);
        *reinterpret_cast<uint4*>(ks + c * 2048 + r * 128 + ((g0 ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(ks + c * 2048 + r * 128 + (((g0 + 1) ^ (r & 7)) << 4)) = hi;
        i8x16_to_16bit<false>(*reinterpret_cast<const uint4*>(vq + r * kD + u * 16), lo, hi);
        *reinterpret_cast<uint4*>(vs + c * 2048 + r * 128 + ((g0 ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(vs + c * 2048 + r * 128 + (((g0 + 1) ^ (r & 7)) << 4)) = hi;
      }
      // the row scales of this lane's accumulator rows (tokens lane / 4, + 8)
      const float* sc = reinterpret_cast<const float*>(smem + slot * Sh::kStageBytes + Sh::kScaleOffset);
      ksc0 = sc[tok0 + (lane >> 2)];
      ksc1 = sc[tok0 + (lane >> 2) + 8];
      vsc0 = sc[Sh::kTok + tok0 + (lane >> 2)];
      vsc1 = sc[Sh::kTok + tok0 + (lane >> 2) + 8];
      __syncwarp();
      // everything this warp needs from the slot is copied out
      if (lane == 0) mbar_arrive(&bars->empty[slot]);
      kbase = smem_u32(ks);
      vbase = smem_u32(vs);
    }
    // ---- S^T = K Q^T ----
    float s[kNT][4];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    if constexpr (kQ4 && Sh::kDirect) {
      // A = K codes as exact fp16, nibbles (i, i + 4) and (i + 1, i + 5) of
      // word kk / 2, i = 2 (kk % 2) (the permutation of the query fragments)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        // (a2, a3: 16 x code, matched by the queries' 1 / 16)
        const int sh = 8 * (kk & 1);
        const uint32_t w0 = kw[0][kk >> 1] >> sh, w1 = kw[1][kk >> 1] >> sh;
        const uint32_t a0 = i4pair_to_f16(w0), a2 = i4pair_hi_to_f16x16(w0);
        const uint32_t a1 = i4pair_to_f16(w1), a3 = i4pair_hi_to_f16x16(w1);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma16816<false>(s[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
      }
    } else if constexpr (Sh::kDirect) {
      // A = K codes as exact fp16: word kk of a row holds d = 32j + 4kk + 0..3
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a0 = i8pair_to_f16(kw[0][kk], false), a2 = i8pair_to_f16(kw[0][kk], true);
        const uint32_t a1 = i8pair_to_f16(kw[1][kk], false), a3 = i8pair_to_f16(kw[1][kk], true);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma16816<false>(s[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
      }
    } else {
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const int mi = lane >> 3, r = lane & 7;
        const int tok = tok0 + (mi & 1) * 8 + r;
        const int c = kk >> 2;
        const int g = (kk & 3) * 2 + (mi >> 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sw128(kbase + c * kTileStride, tok - trow0, g), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma16816<kBF16>(s[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
      }
    }
    // ---- logits, mask, online softmax ----
    const int wtok = (t_begin + i) * Sh::kTok + tok0;  // first token of this warp's 16
    // token of s[.][0], s[.][1] (s[.][2], s[.][3]: + 8)
    const int pos0 = wtok + ((kQ4 && Sh::kDirect) ? i4_token(lane >> 2) : (lane >> 2));
    // every column sees all 16 tokens: no mask (warp-uniform)
    const bool all_visible = wtok >= lo_in && wtok + 16 <= hi_in;
    float vr = 1.f;
    if constexpr (kQuant) {
      // S^T rows are tokens: the K scale multiplies each row (and, direct
      // path, 2^e of the column undoes the query scaling)
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        s[nt][0] *= ksc0 * qsc[nt][0];
        s[nt][1] *= ksc0 * qsc[nt][1];
        s[nt][2] *= ksc1 * qsc[nt][0];
        s[nt][3] *= ksc1 * qsc[nt][1];
      }
      // slots at positions >= Lk may hold any scale (NaN included): their P
      // is 0 and must stay 0 after the V scale is folded in
      if (wtok + 16 > Lk) {
        if (pos0 >= Lk) vsc0 = 0.f;
        if (pos0 + 8 >= Lk) vsc1 = 0.f;
      }
      // the warp's largest V scale (the four lanes of a row hold the same
      // two scales); vC and its reciprocal change only when it grows
      float c = fmaxf(vsc0, vsc1);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, off));
      if (c > vC) {
        const float inv = 1.f / c;
        vr = vC * inv;  // acc (in units of vC) -> units of c
        vC = c;
        vCinv = inv;
      }
      vsc0 *= vCinv;
      vsc1 *= vCinv;
    }
    uint32_t pb[kNT][2];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      float x0 = dec_logit(s[nt][0], p);
      float x1 = dec_logit(s[nt][1], p);
      float x2 = dec_logit(s[nt][2], p);
      float x3 = dec_logit(s[nt][3], p);
      if (alibi) {  // -slope * |query - key|, after softcap
        const float pf = static_cast<float>(pos0);
        x0 = fmaf(-asl[nt][0], fabsf(aqp[nt][0] - pf), x0);
        x1 = fmaf(-asl[nt][1], fabsf(aqp[nt][1] - pf), x1);
        x2 = fmaf(-asl[nt][0], fabsf(aqp[nt][0] - pf - 8.f), x2);
        x3 = fmaf(-asl[nt][1], fabsf(aqp[nt][1] - pf - 8.f), x3);
      }
      if (!all_visible) {
        // per-column key ranges (padding columns take the last real one's)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int n = min(n0 + nt * 8 + 2 * (lane & 3) + j, p.n_cols - 1);
          const int qpos = qbase + n / p.group;
          const int clo = key_lo(p, qpos), chi = key_hi(p, qpos, Lk);
          if (pos0 < clo || pos0 >= chi) (j ? x1 : x0) = -INFINITY;
          if (pos0 + 8 < clo || pos0 + 8 >= chi) (j ? x3 : x2) = -INFINITY;
        }
      }
      // column maxima over the warp's 16 tokens: reduce over lane >> 2
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
      const float al0 = mn0 == -INFINITY ? 1.f : ex2_approx(m_run[nt][0] - mn0);
      const float al1 = mn1 == -INFINITY ? 1.f : ex2_approx(m_run[nt][1] - mn1);
      m_run[nt][0] = mn0;
      m_run[nt][1] = mn1;
      const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
      const float e0 = ex2_approx(x0 - b0), e1 = ex2_approx(x1 - b1);
      const float e2 = ex2_approx(x2 - b0), e3 = ex2_approx(x3 - b1);
      l_part[nt][0] = l_part[nt][0] * al0 + e0 + e2;
      l_part[nt][1] = l_part[nt][1] * al1 + e1 + e3;
      const float ar0 = al0 * vr, ar1 = al1 * vr;
      // (warp-uniform: most slices move neither the max nor vC)
      if (__any_sync(0xffffffffu, ar0 != 1.f || ar1 != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < kD / 16; ++mt) {
          acc[nt][mt][0] *= ar0;
          acc[nt][mt][1] *= ar1;
          acc[nt][mt][2] *= ar0;
          acc[nt][mt][3] *= ar1;
        }
      }
      // P^T fragments: transpose the two 8x8 blocks of the 16x8 accumulator
      // (int8: the V row scale folded into P, token by token)
      if constexpr (kQuant) {
        pb[nt][0] = movmatrix_t(pack2<false>(e0 * vsc0, e1 * vsc0));
        pb[nt][1] = movmatrix_t(pack2<false>(e2 * vsc1, e3 * vsc1));
      } else {
        pb[nt][0] = movmatrix_t(pack2<kBF16>(e0, e1));
        pb[nt][1] = movmatrix_t(pack2<kBF16>(e2, e3));
      }
    }
    // ---- O^T += V^T P^T ----
    if constexpr (kQ4 && Sh::kDirect) {
      // A = V^T codes as exact fp16; accumulator rows r, r + 8 of step mt are
      // d = 16r + 2mt and 16r + 2mt + 1, the low and high nibble of byte mt of
      // this lane's V words; byte b of tokens 2j, 2j+1 (2j+8, 2j+9) is brought
      // to bytes 0 and 2 first
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const uint32_t bsel = static_cast<uint32_t>(mt & 3);
        const uint32_t sel = bsel | ((bsel + 4) << 8);
        const uint32_t x = __byte_perm(vw[0][mt >> 2], vw[1][mt >> 2], sel);
        const uint32_t y = __byte_perm(vw[2][mt >> 2], vw[3][mt >> 2], sel);
        // rows r + 8 (odd d) as 16 x code: the epilogue divides them by 16
        const uint32_t a0 = i4pair_to_f16(x), a1 = i4pair_hi_to_f16x16(x);
        const uint32_t a2 = i4pair_to_f16(y), a3 = i4pair_hi_to_f16x16(y);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma16816<false>(acc[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    } else if constexpr (Sh::kDirect) {
      // A = V^T codes as exact fp16; accumulator rows r, r + 8 of step mt are
      // d = 16r + 2mt and 16r + 2mt + 1 (bytes 2mt, 2mt + 1 of this lane's V
      // words); k = tokens 2j, 2j+1 (a0, a1) and 2j+8, 2j+9 (a2, a3)
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const uint32_t o = 2 * (mt & 1);
        const uint32_t sel = o | ((o + 4) << 4) | ((o + 1) << 8) | ((o + 5) << 12);
        const uint32_t x = __byte_perm(vw[0][mt >> 1], vw[1][mt >> 1], sel);
        const uint32_t y = __byte_perm(vw[2][mt >> 1], vw[3][mt >> 1], sel);
        const uint32_t a0 = i8pair_to_f16(x, false), a1 = i8pair_to_f16(x, true);
        const uint32_t a2 = i8pair_to_f16(y, false), a3 = i8pair_to_f16(y, true);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma16816<false>(acc[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    } else {
      // Slots at positions >= Lk (the rest of the last page, or the next
      // sequence of a contiguous cache) may hold anything, NaN included; P is 0
      // there but 0 * NaN is not, so those V elements are zeroed. Fragment
      // registers a0, a1 hold tokens wtok + 2*(lane&3) + {0, 1} (low, high
      // half), a2, a3 the same tokens + 8.
      const bool tail = wtok + 16 > Lk;  // warp-uniform
      uint32_t vm01 = 0xffffffffu, vm23 = 0xffffffffu;
      if (tail) {
        const int k0 = wtok + 2 * (lane & 3);
        vm01 = (k0 < Lk ? 0x0000ffffu : 0u) | (k0 + 1 < Lk ? 0xffff0000u : 0u);
        vm23 = (k0 + 8 < Lk ? 0x0000ffffu : 0u) | (k0 + 9 < Lk ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int mt = 0; mt < kD / 16; ++mt) {
        const int mi = lane >> 3, r = lane & 7;
        const int tok = tok0 + (mi >> 1) * 8 + r;
        const int dcol = mt * 16 + (mi & 1) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(sw128(vbase + (dcol >> 6) * kTileStride, tok - trow0, (dcol & 63) >> 3), a0, a1, a2, a3);
        if (tail) {
          a0 &= vm01;
          a1 &= vm01;
          a2 &= vm23;
          a3 &= vm23;
        }
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
          mma16816<kBF16 && !kQuant>(acc[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    }
    __syncwarp();
    if (!kQuant && lane == 0) mbar_arrive(&bars->empty[slot]);
  }

  // ---- merge the four warps' states, then write the split's result ----
  // per warp and column: m (log2 domain), l; per column and d: unnormalised O
  named_bar_sync(1, 128);  // every consumer is done reading the stage ring
  float* red_m = red;                        // [4][kH]
  float* red_l = red + 4 * kH;               // [4][kH]
  float* red_o = red + 8 * kH;               // [4][kH][kD]
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
    float l0 = l_part[nt][0], l1 = l_part[nt][1];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const int h0 = nt * 8 + 2 * (lane & 3);
    if (lane < 4) {
      red_m[warp * kH + h0] = m_run[nt][0];
      red_m[warp * kH + h0 + 1] = m_run[nt][1];
      red_l[warp * kH + h0] = l0;
      red_l[warp * kH + h0 + 1] = l1;
    }
    const float oc = kQuant ? vC : 1.f;  // int8 / int4: acc holds O / vC
    const float oc1 = (kQ4 && Sh::kDirect) ? oc * 0.0625f : oc;  // int4, D = 128: rows d1 hold 16 O / vC
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt) {
      // accumulator rows lane / 4 and lane / 4 + 8 of step mt
      const int d0 = Sh::kDirect ? 16 * (lane >> 2) + 2 * mt : mt * 16 + (lane >> 2);
      const int d1 = Sh::kDirect ? d0 + 1 : d0 + 8;
      red_o[(warp * kH + h0) * kD + d0] = acc[nt][mt][0] * oc;
      red_o[(warp * kH + h0 + 1) * kD + d0] = acc[nt][mt][1] * oc;
      red_o[(warp * kH + h0) * kD + d1] = acc[nt][mt][2] * oc1;
      red_o[(warp * kH + h0 + 1) * kD + d1] = acc[nt][mt][3] * oc1;
    }
  }
  named_bar_sync(1, 128);
  // 128 threads: each (column, d) combination
  for (int idx = threadIdx.x; idx < n_here * kD; idx += 128) {
    const int c = idx / kD, d = idx % kD;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) m = fmaxf(m, red_m[w * kH + c]);
    float l = 0.f, o = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float sc = ex2_approx(red_m[w * kH + c] - m);
        l += red_l[w * kH + c] * sc;
        o += red_o[(w * kH + c) * kD + d] * sc;
      }
    }
    const float on = l > 0.f ? o / l : 0.f;
    const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    const int n = n0 + c;
    const int t = n / p.group;
    const int hq = kvh * p.group + n % p.group;
    const size_t row = (static_cast<size_t>(b) * p.Sq + t) * p.Hq + hq;  // row of out
    if (p.splits == 1) {
      const size_t oi = row * kD + d;
      if constexpr (kBF16)
        static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(on);
      else
        static_cast<__half*>(p.out)[oi] = __float2half_rn(on);
      if (d == 0) p.lse[(static_cast<size_t>(b) * p.Hq + hq) * p.Sq + t] = lse;
    } else {
      const size_t pi = static_cast<size_t>(split) * p.B * p.Sq * p.Hq + row;
      p.part_o[pi * kD + d] = on;
      if (d == 0) p.part_lse[pi] = lse;
    }
  }
  __syncthreads();
}

// one warp per output row (b, t, hq): merge the splits' partials
template <int kD, bool kBF16>
__global__ void lse_combine_kernel(const DecodeParams p) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const size_t stride = static_cast<size_t>(p.B) * p.Sq * p.Hq;
  if (gw >= stride) return;
  float m = -INFINITY;
  for (int s = 0; s < p.splits; ++s) m = fmaxf(m, p.part_lse[s * stride + gw]);
  float wsum = 0.f;
  float o[kD / 32];
#pragma unroll
  for (int j = 0; j < kD / 32; ++j) o[j] = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const float ls = p.part_lse[s * stride + gw];
      const float w = __expf(ls - m);
      wsum += w;
      const float* po = p.part_o + (s * stride + gw) * kD;
#pragma unroll
      for (int j = 0; j < kD / 32; ++j) o[j] += w * po[j * 32 + lane];
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int j = 0; j < kD / 32; ++j) {
    const size_t oi = static_cast<size_t>(gw) * kD + j * 32 + lane;
    if constexpr (kBF16)
      static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o[j] * inv);
    else
      static_cast<__half*>(p.out)[oi] = __float2half_rn(o[j] * inv);
  }
  if (lane == 0) {
    const int hq = gw % p.Hq, t = (gw / p.Hq) % p.Sq, b = gw / (p.Hq * p.Sq);
    p.lse[(static_cast<size_t>(b) * p.Hq + hq) * p.Sq + t] = wsum > 0.f ? m + __logf(wsum) : -INFINITY;
  }
}

}  // namespace fa
