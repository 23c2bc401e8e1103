// Backward attention kernels for sm_100a. The attention matrix is never
// stored: P is recomputed from Q, K and the saved LSE ("FlashAttention 实战指南"
// §长序列注意力为什么会爆内存: the backward pass recomputes the attention
// matrix when it needs it instead of keeping it).
//
// With P the softmax probabilities of the forward pass,
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dO * O)),
//   dQ = scale * dS K,  dK = scale * dS^T Q
// (and dS picks up the factor 1 - tanh^2 under softcap).
//
//   bwd_pre_kernel   Drow = rowsum(dO * O) and -LSE (exp2 domain) per
//                    (token, query head), into a padded per-row layout.
//   bwd_dkdv_kernel  one CTA per (sequence, kv head, 128-key tile): K and V
//                    stay resident while the CTA walks every query head of the
//                    GQA group and every 64-row query block that can see the
//                    keys; dK and dV accumulate in tensor memory (no atomics).
//   bwd_dq_kernel    one CTA per (sequence, query head, 128-row Q tile): Q and
//                    dO stay resident in shared memory while the CTA walks the
//                    visible 128-key K/V blocks; dQ accumulates in tensor
//                    memory and is written once (no atomics, so the whole
//                    backward is deterministic).
//   bwd_dkdv_pass_kernel, bwd_dq256_kernel: the same two halves at D = 256,
//                    where the accumulators leave less tensor memory.
// dS is computed in both kernels (S and dP are recomputed twice): seven
// 128x128xD products per (query tile, key tile) instead of five, in exchange
// for no dQ reduction across CTAs and a pipeline with no write-back on the
// critical path.
//
// bwd_dkdv warp roles (608 threads); an item is one (query head, 64-row
// query block) against the CTA's 128 keys:
//   warp 0      TMA producer: K, V once; Q_i, dO_i and the rows' -LSE and Drow
//               into a 4-slot ring.
//   warp 1      MMA issuer of S^T and dV (one lane), TMEM owner.
//   warp 2      MMA issuer of dP^T and dK (one lane).
//   warps 3-18  two teams of two compute groups; team t takes the items with
//               i % 2 == t, group g of a team the item's query columns
//               [32g, 32g+32): one thread per key row computes
//               P^T = exp(S^T - LSE) and then dS^T = P^T * (dP^T - Drow), each
//               written back to TMEM as 16-bit pairs over the first half of
//               the columns it came from, where the dV and dK MMAs read their
//               A operand. While one team computes, the tensor core runs the
//               other team's MMAs. At the end warps 3-10 write dV, 11-18 dK.
// TMEM columns: A_t [64t, 64t+64) S^T then P^T; B_t [128+64t, +64) dP^T then
// dS^T (queries [32g, 32g+32) packed into [32g, 32g+16) of each);
// dV [256, 256+D); dK [256+D, 256+2D).
// MMA order per item i (team t = i % 2): dV_i, S_{i+2} -> A_t, dK_i,
// dP_{i+2} -> B_t.
#pragma once

#include "ptx.cuh"

namespace fa {

struct BwdParams {
  int B, Hq, Hkv, S, total, group;
  int n_ktiles;              // ceil(S / 128)
  float scale;               // multiplies dK and dQ in the epilogues
  float scale_log2;          // scale * log2(e)
  float softcap, cap_in, cap_out_log2;
  int wl, wr;                // window (causal folded into wr)
  const void* q;
  const void* o;
  const void* dout;
  const float* lse;          // forward LSE, (B, Hq, S) or (Hq, total)
  float* vec_nlse;           // -LSE * log2(e) (-inf for an empty row), padded layout
  float* vec_drow;           // rowsum(dO * O), padded layout
  int tpad;                  // per-head stride of the padded layout
  void* dq;                  // (T, Hq, D) 16-bit
  void* dk;                  // (T, Hkv, D)
  void* dv;
  const int* cu_seqlens;
  const float* alibi;        // ALiBi slopes, nullable: slope of (b, h) = alibi[b * alibi_bstride + h]
  int alibi_bstride;
  // elements from one token's row to the next: q and dq (Hq * D unpacked),
  // dk and dv (Hkv * D unpacked); the qkv-packed layout uses 3 * H * D
  long long q_tok, dq_tok, dkv_tok;
};

// ALiBi slope of (sequence b, query head h) in the exp2 domain, 0 without ALiBi
__device__ __forceinline__ float alibi_slope2(const BwdParams& p, int b, int h) {
  return p.alibi ? p.alibi[static_cast<size_t>(b) * p.alibi_bstride + h] * 1.4426950408889634f : 0.f;
}

// Padded layout of the per-row vectors: query row q of sequence b (first
// token seq_start) and query head h sits at
//   h * tpad + 128 * (seq_start / 128 + b) + q,  tpad = 128 * (T / 128 + B + 1).
// Each 128-row tile of a sequence is then contiguous and 512-byte aligned (one
// bulk copy), and the tiles of different sequences never overlap:
// seq_start / 128 + ceil(len / 128) <= (seq_start + len) / 128 + 1.
__device__ __forceinline__ size_t vec_index(const BwdParams& p, int h, int b, int seq_start, int q) {
  return static_cast<size_t>(h) * p.tpad + 128 * static_cast<size_t>(seq_start / 128 + b) + q;
}

// ---------------------------------------------------------------------------
// pre: Drow = rowsum(dO * O) and -LSE in the exp2 domain, both into the padded
// layout. A block takes tpb consecutive tokens with all their heads
// (tpb * Hq rows of the (token, head)-major O and dO, one contiguous range) and
// reads them in order: kLanes lanes per row, 16 bytes of O and of dO each,
// kIter rows per lane group with their loads issued together. The row sums go
// to shared memory; the block then writes both vectors head by head, tpb
// consecutive entries each. Index arithmetic is 32-bit within a block.
// ---------------------------------------------------------------------------
template <int kD>
struct PreShape {
  static constexpr int kThreads = 256;
  static constexpr int kLanes = kD / 8;
  static constexpr int kRowsPerWarp = 32 / kLanes;  // rows a warp reads at a time
  static constexpr int kIter = 4;                   // of those, per lane group in flight
};
constexpr int kPreRowsPerBlock = 512;  // rows a block covers (at least one token)
constexpr int kPreMaxHeads = 8192;     // keeps one token's row sums within 48 KB of shared memory

// tokens per block, and the dynamic shared memory that takes
inline int pre_tokens_per_block(int Hq) { return Hq >= kPreRowsPerBlock ? 1 : kPreRowsPerBlock / Hq; }
inline size_t pre_smem_bytes(int Hq) {
  const int tpb = pre_tokens_per_block(Hq);
  return (static_cast<size_t>(tpb) * Hq + 2 * static_cast<size_t>(tpb)) * sizeof(float);
}

template <int kD, bool kBF16>
__global__ void __launch_bounds__(PreShape<kD>::kThreads) bwd_pre_kernel(const BwdParams p, int tpb) {
  using Sh = PreShape<kD>;
  extern __shared__ float pre_smem[];
  const int tok0 = static_cast<int>(blockIdx.x) * tpb;
  const int ntok = min(tpb, p.total - tok0);
  const uint32_t nrows = static_cast<uint32_t>(ntok) * static_cast<uint32_t>(p.Hq);
  float* s_acc = pre_smem;                                    // [ntok][Hq]
  int* s_b = reinterpret_cast<int*>(pre_smem + static_cast<size_t>(tpb) * p.Hq);  // sequence of a token
  int* s_start = s_b + tpb;                                   // and its first token
  for (int tl = threadIdx.x; tl < ntok; tl += Sh::kThreads) {
    const int tok = tok0 + tl;
    int b;
    if (p.cu_seqlens != nullptr) {
      // the largest b with cu_seqlens[b] <= tok
      int lo = 0, hi = p.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cu_seqlens[mid] <= tok)
          lo = mid;
        else
          hi = mid - 1;
      }
      b = lo;
      s_start[tl] = p.cu_seqlens[b];
    } else {
      b = tok / p.S;
      s_start[tl] = b * p.S;
    }
    s_b[tl] = b;
  }
  // ---- row sums, reading the block's range in order ----
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int li = lane % Sh::kLanes;
  constexpr uint32_t kWarpRows = Sh::kRowsPerWarp * Sh::kIter;
  constexpr uint32_t kStride = kWarpRows * (Sh::kThreads / 32);
  const uint16_t* o_blk = static_cast<const uint16_t*>(p.o) + static_cast<size_t>(tok0) * p.Hq * kD;
  const uint16_t* d_blk = static_cast<const uint16_t*>(p.dout) + static_cast<size_t>(tok0) * p.Hq * kD;
  // (the loop bound depends on the warp only, so every lane takes part in
  // the shuffles)
  for (uint32_t rb = warp * kWarpRows; rb < nrows; rb += kStride) {
    uint4 ov[Sh::kIter], dv[Sh::kIter];
#pragma unroll
    for (int k = 0; k < Sh::kIter; ++k) {
      const uint32_t r = rb + k * Sh::kRowsPerWarp + lane / Sh::kLanes;
      ov[k] = dv[k] = make_uint4(0u, 0u, 0u, 0u);
      if (r < nrows) {
        ov[k] = *reinterpret_cast<const uint4*>(o_blk + r * kD + li * 8);
        dv[k] = *reinterpret_cast<const uint4*>(d_blk + r * kD + li * 8);
      }
    }
#pragma unroll
    for (int k = 0; k < Sh::kIter; ++k) {
      const uint32_t ow[4] = {ov[k].x, ov[k].y, ov[k].z, ov[k].w}, dw[4] = {dv[k].x, dv[k].y, dv[k].z, dv[k].w};
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 o2 = unpack2<kBF16>(ow[i]), d2 = unpack2<kBF16>(dw[i]);
        acc = fmaf(o2.x, d2.x, fmaf(o2.y, d2.y, acc));
      }
#pragma unroll
      for (int off = Sh::kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const uint32_t r = rb + k * Sh::kRowsPerWarp + lane / Sh::kLanes;
      if (li == 0 && r < nrows) s_acc[r] = acc;
    }
  }
  __syncthreads();
  // ---- both vectors, head by head: consecutive threads take consecutive
  // tokens of one head ----
  for (uint32_t i = threadIdx.x; i < nrows; i += Sh::kThreads) {
    const int h = static_cast<int>(i / static_cast<uint32_t>(ntok));
    const int tl = static_cast<int>(i - static_cast<uint32_t>(h) * static_cast<uint32_t>(ntok));
    const int tok = tok0 + tl, b = s_b[tl], seq_start = s_start[tl];
    const size_t lidx = p.cu_seqlens != nullptr
                            ? static_cast<size_t>(h) * p.total + tok
                            : (static_cast<size_t>(b) * p.Hq + h) * p.S + (tok - seq_start);
    const float l = p.lse[lidx];
    const size_t vi = vec_index(p, h, b, seq_start, tok - seq_start);
    p.vec_nlse[vi] = (l == -INFINITY) ? -INFINITY : -l * 1.4426950408889634f;
    p.vec_drow[vi] = s_acc[static_cast<uint32_t>(tl) * static_cast<uint32_t>(p.Hq) + h];
  }
}

// site: 100 * kernel (1 dK/dV, 2 dV pass, 3 dK pass, 4 dQ) + wait, recorded
// when this wait is the one that gives up
__device__ __forceinline__ bool bwd_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         int site = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        record_timeout(site);
        *abort = 1;
        return false;
      }
    }
  }
}

// For a pair of raw scores s = q.k: the exponent of P in the exp2 domain,
// x = logit * log2(e) - LSE * log2(e) (nl2 holds the second term), and the
// factor dS picks up from the softcap, 1 - tanh^2 (1 without softcap). The
// common factor `scale` of dS is applied to dK and dQ in the epilogues.
template <bool kCap>
__device__ __forceinline__ void bwd_logit2(float2 s2, bool poly, const BwdParams& p, float2 nl2,
                                           float2& x, float2& fac) {
  if constexpr (kCap) {
    float2 th;
    if (poly)
      th = tanh_poly2(__fmul2_rn(s2, make_float2(p.cap_in, p.cap_in)));
    else
      th = make_float2(tanh_fast(s2.x * p.cap_in), tanh_fast(s2.y * p.cap_in));
    x = __ffma2_rn(th, make_float2(p.cap_out_log2, p.cap_out_log2), nl2);
    fac = __ffma2_rn(make_float2(-th.x, -th.y), th, make_float2(1.f, 1.f));
  } else {
    x = __ffma2_rn(s2, make_float2(p.scale_log2, p.scale_log2), nl2);
    fac = make_float2(1.f, 1.f);
  }
}

// is every |scale * s / softcap| of these 32 raw scores, in every lane of
// the warp, small enough for the tanh polynomial?
__device__ __forceinline__ bool poly_ok(const uint32_t (&sr)[32], float cap_in) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2)
    amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(sr[i])), fabsf(__uint_as_float(sr[i + 1]))));
  return __all_sync(0xffffffffu, amax * fabsf(cap_in) <= kTanhPolyMax);
}

// ALiBi for 32 entries: w[i] -= sl2 * |d0 + sgn * i| (sl2: slope in the exp2
// domain). When the sign of d0 + sgn * i is the same for all 32 entries in
// every lane of the warp (`one_side`: always, for the visible pairs of a
// causal mask), |.| is affine in i and one packed FMA per pair adds it.
__device__ __forceinline__ void alibi32(float (&w)[32], float sl2, float d0, float sgn,
                                        bool one_side) {
  const float last = d0 + sgn * 31.f;
  const bool pos = d0 >= 0.f && last >= 0.f, neg = d0 <= 0.f && last <= 0.f;
  if (__all_sync(0xffffffffu, one_side || pos || neg)) {
    // one_side: the visible pairs have d0 + sgn i >= 0 (masked ones are zeroed later)
    const float s = (one_side || pos) ? -sl2 : sl2;
    const float2 c2 = make_float2(s * d0, s * d0), d2 = make_float2(s * sgn, s * sgn);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 b = __ffma2_rn(make_float2(static_cast<float>(i), static_cast<float>(i + 1)), d2, c2);
      const float2 v = __fadd2_rn(make_float2(w[i], w[i + 1]), b);
      w[i] = v.x;
      w[i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = fmaf(-sl2, fabsf(d0 + sgn * static_cast<float>(i)), w[i]);
  }
}

// P (or P * (1 - tanh^2) under softcap) of 32 raw scores sharing one -LSE
// (nl2, in the exp2 domain): all exponentials are issued before any result
// is consumed, so they pipeline through the special-function unit. With
// ALiBi, entry i gets -sl2 * |d0 - i| added to its exponent (sl2: slope in
// the exp2 domain, d0: query position minus the first key's).
// kPolyOf8: of every 8 pairs of exponentials, this many run as an FMA-pipe
// cubic instead of on the special-function unit.
template <bool kCap, int kPolyOf8 = 0>
__device__ __forceinline__ void bwd_probs32(uint32_t (&sr)[32], float2 nl2, const BwdParams& p,
                                            bool alibi, float sl2, float d0, float (&w)[32],
                                            bool causal_side) {
  const bool poly = kCap ? poly_ok(sr, p.cap_in) : false;
#pragma unroll
  for (int j2 = 0; j2 < 16; ++j2) {
    const float2 s2 = make_float2(__uint_as_float(sr[2 * j2]), __uint_as_float(sr[2 * j2 + 1]));
    float2 x, fac;
    bwd_logit2<kCap>(s2, poly, p, nl2, x, fac);
    w[2 * j2] = x.x;
    w[2 * j2 + 1] = x.y;
    if constexpr (kCap) {  // the raw scores are no longer needed
      sr[2 * j2] = __float_as_uint(fac.x);
      sr[2 * j2 + 1] = __float_as_uint(fac.y);
    }
  }
  if (alibi) alibi32(w, sl2, d0, -1.f, causal_side);
#pragma unroll
  for (int j2 = 0; j2 < 16; ++j2) {
    if ((j2 & 7) < kPolyOf8) {
      const float2 e = ex2_poly2(make_float2(w[2 * j2], w[2 * j2 + 1]));
      w[2 * j2] = e.x;
      w[2 * j2 + 1] = e.y;
    } else {
      w[2 * j2] = ex2_approx(w[2 * j2]);
      w[2 * j2 + 1] = ex2_approx(w[2 * j2 + 1]);
    }
  }
  if constexpr (kCap) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] *= __uint_as_float(sr[i]);
  }
}

// ===========================================================================
// dK, dV
// ===========================================================================
// kPass: which gradients one launch computes. D <= 128: both (kDkdvBoth),
// their accumulators side by side in TMEM. D = 256: dV and dK alone take all
// 512 TMEM columns ("FlashAttention 实战指南" §版本怎么选 allows head dims up
// to 256), so the host runs a dV pass (S^T, P^T, dV += P^T dO; K resident, no
// V) and then a dK pass (S^T, dP^T, dS^T, dK += dS^T Q; P stays in
// registers). Each pass recomputes S^T; the two cost 10 D per pair against 8 D
// for the fused kernel. At D = 256 an item is 32 query rows (one compute
// group per team), so that K and V (64 KB each) and three Q/dO slots fit in
// shared memory.
enum : int { kDkdvBoth = 0, kDvOnly = 1, kDkOnly = 2 };

template <int kD, int kPass = kDkdvBoth>
struct DkdvShape {
  static_assert((kPass == kDkdvBoth) == (kD <= 128), "D <= 128 fuses dK and dV; D = 256 splits them");
  static constexpr int kChunks = kD / 64;
  static constexpr int kChunkBytes = 128 * 128;        // K/V: 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kQRows = kD == 256 ? 32 : 64;   // query rows per item
  static constexpr int kGroups = kQRows / 32;          // compute groups per team
  static constexpr int kQChunkBytes = kQRows * 128;
  static constexpr int kQTileBytes = kChunks * kQChunkBytes;
  static constexpr bool kNeedV = kPass != kDvOnly;
  static constexpr int kSlots = kD == 256 ? (kNeedV ? 3 : 5) : 4;  // Q/dO ring
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = (kNeedV ? 2 : 1) * kTileBytes;  // + slot * 2 * kQTileBytes (Q, dO)
  // per slot: -LSE (exp2 domain)[kQRows], Drow[kQRows] of the slot's query rows
  static constexpr int kOffVec = kOffQ + kSlots * 2 * kQTileBytes;
  static constexpr int kVecBytes = 2 * kQRows * 4;
  static constexpr int kOffBar = kOffVec + kSlots * kVecBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
  // warp 0 TMA, warps 1 .. kIssuers MMA, then two teams of kGroups compute
  // groups (4 warps each); team t takes the items it with it % 2 == t, group
  // g of a team the 32 query columns [32g, 32g + 32) of the item. The fused
  // kernel issues from two threads (one tcgen05.mma with N = 64 takes about
  // as long to issue as to run): warp 1 the S^T and dV products, warp 2 the
  // dP^T and dK ones.
  static constexpr int kIssuers = kPass == kDkdvBoth ? 2 : 1;
  static constexpr int kFirst = 1 + kIssuers;  // first compute warp
  static constexpr int kThreads = 32 * kFirst + 2 * kGroups * 128;
  static constexpr int kTmemCols = 512;
  static constexpr int kColA = 0;             // + kQRows t: team t's S^T, then P^T
  static constexpr int kColB = 2 * kQRows;    // + kQRows t: team t's dP^T, then dS^T
  static constexpr int kColDV = kPass == kDkdvBoth ? 256 : 256;
  static constexpr int kColDK = kPass == kDkdvBoth ? 256 + kD : 256;
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB a CTA may use");
  static_assert(kSlots <= 8, "more ring slots than the barrier block holds");
};

struct DkdvBars {
  uint64_t kv_full;
  uint64_t qd_full[8];   // one per ring slot (DkdvShape::kSlots <= 8)
  uint64_t qd_empty[8];
  uint64_t s_ready[2];   // per team
  uint64_t dp_ready[2];
  uint64_t p_ready[2];
  uint64_t ds_ready[2];
  uint64_t final_done;   // one commit per issuer
  uint64_t drain[2];     // per issuer
  uint32_t tmem_base;
  int abort;
};

template <int kD, bool kBF16, bool kCap, bool kAlibi, int kPass = kDkdvBoth>
__global__ void __launch_bounds__(DkdvShape<kD, kPass>::kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  using Sh = DkdvShape<kD, kPass>;
  constexpr int kSite = 100 * (1 + kPass);  // wait sites of this kernel (bwd_wait)
  constexpr bool kDoDV = kPass != kDkOnly;  // this launch accumulates dV
  constexpr bool kDoDK = kPass != kDvOnly;  // and dK
  static_assert(sizeof(DkdvBars) <= Sh::kBarBytes, "barrier block exceeds its reservation");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DkdvBars* bars = reinterpret_cast<DkdvBars*>(smem + Sh::kOffBar);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (sequence, kv head) major; within a head, key tiles in
  // increasing order (under causal masking the first ones see the most rows)
  const int bk = static_cast<int>(blockIdx.x) / p.n_ktiles;
  const int kt = static_cast<int>(blockIdx.x) % p.n_ktiles;
  const int kvh = bk % p.Hkv;
  const int b = bk / p.Hkv;
  int seq_start, seq_len;
  if (p.cu_seqlens != nullptr) {
    seq_start = p.cu_seqlens[b];
    seq_len = p.cu_seqlens[b + 1] - seq_start;
  } else {
    seq_start = b * p.S;
    seq_len = p.S;
  }
  const int k0 = kt * 128;
  if (k0 >= seq_len) return;
  // query rows that can see some key of [k0, k0 + 127], in 64-row blocks
  int q_lo = 0;
  if (p.wr >= 0) q_lo = max(0, k0 - p.wr);
  int q_hi = seq_len - 1;
  if (p.wl >= 0) q_hi = min(q_hi, k0 + 127 + p.wl);
  const int i_begin = q_lo / Sh::kQRows;
  const int i_cnt = q_hi >= q_lo ? q_hi / Sh::kQRows + 1 - i_begin : 0;
  const int n_items = i_cnt * p.group;  // (head, 64-row query block) pairs
  // item it's Q and dO tiles and row vectors into ring slot it % kSlots
  auto load_qd = [&](int it) {
    const int slot = it % Sh::kSlots;
    const int h = kvh * p.group + it / i_cnt;
    const int q0 = (i_begin + it % i_cnt) * Sh::kQRows;
    const int tok = seq_start + q0;
    uint8_t* dst = smem + Sh::kOffQ + slot * 2 * Sh::kQTileBytes;
    uint8_t* vdst = smem + Sh::kOffVec + slot * Sh::kVecBytes;
    const size_t vi = vec_index(p, h, b, seq_start, q0);
    mbar_arrive_expect_tx(&bars->qd_full[slot], 2 * Sh::kQTileBytes + Sh::kVecBytes);
    for (int c = 0; c < Sh::kChunks; ++c) {
      tma_load_3d(&tm_q, &bars->qd_full[slot], dst + c * Sh::kQChunkBytes, c * 64, h, tok);
      tma_load_3d(&tm_do, &bars->qd_full[slot], dst + Sh::kQTileBytes + c * Sh::kQChunkBytes, c * 64,
                  h, tok);
    }
    // the rows' vectors (rows past the sequence end hold stale values; the
    // compute groups mask those columns)
    bulk_load(vdst, p.vec_nlse + vi, Sh::kVecBytes / 2, &bars->qd_full[slot]);
    bulk_load(vdst + Sh::kVecBytes / 2, p.vec_drow + vi, Sh::kVecBytes / 2, &bars->qd_full[slot]);
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < Sh::kSlots; ++s) {
      mbar_init(&bars->qd_full[s], 1);
      mbar_init(&bars->qd_empty[s], Sh::kIssuers);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_ready[t], 1);
      mbar_init(&bars->dp_ready[t], 1);
      mbar_init(&bars->p_ready[t], 4 * Sh::kGroups);
      mbar_init(&bars->ds_ready[t], 4 * Sh::kGroups);
      mbar_init(&bars->drain[t], 1);
    }
    mbar_init(&bars->final_done, Sh::kIssuers);
    bars->abort = 0;
    fence_mbar_init();
    // the key block and the first item are requested here, so that their
    // latency overlaps the TMEM allocation and the block sync below
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    mbar_arrive_expect_tx(&bars->kv_full, (Sh::kNeedV ? 2 : 1) * Sh::kTileBytes);
    for (int c = 0; c < Sh::kChunks; ++c) {
      tma_load_3d(&tm_k, &bars->kv_full, smem + Sh::kOffK + c * Sh::kChunkBytes, c * 64, kvh,
                  seq_start + k0);
      if constexpr (Sh::kNeedV)
        tma_load_3d(&tm_v, &bars->kv_full, smem + Sh::kOffV + c * Sh::kChunkBytes, c * 64, kvh,
                    seq_start + k0);
    }
    if (n_items > 0) load_qd(0);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, Sh::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (elect_one()) {
      // (the key block and item 0 were requested at setup)
      int it = n_items > 0 ? 1 : 0;
      for (; it < n_items && !*abort; ++it) {
        const int slot = it % Sh::kSlots;
        const uint32_t ph = static_cast<uint32_t>(it / Sh::kSlots) & 1u;
        if (!bwd_wait(&bars->qd_empty[slot], ph ^ 1u, abort, kSite + 1)) break;
        load_qd(it);
      }
      for (int f = max(0, it - Sh::kSlots); f < it; ++f)
        mbar_wait(&bars->qd_full[f % Sh::kSlots], static_cast<uint32_t>(f / Sh::kSlots) & 1u, kWaitTimeoutNs, kSite + 10);
      mbar_wait(&bars->kv_full, 0, kWaitTimeoutNs, kSite + 11);
    }
    __syncwarp();
  } else if (warp <= Sh::kIssuers) {
    // ======================= MMA issuers =======================
    // Issue order per item i (team t = i % 2, regions A_t, B_t):
    //   dV_i (after the P pass of i), S_{i+2} -> A_t, dK_i (after the dS pass
    //   of i), dP_{i+2} -> B_t.
    // S_{i+2} overwrites A_t only after dV_i, its last reader, in issue
    // order; dP_{i+2} overwrites B_t after dK_i. With two issuers the first
    // runs the A chain (S, dV) and the second the B chain (dP, dK): each
    // region is written and read by one thread, whose products run in issue
    // order, and no product reads the other chain's region. The other
    // team's item i+1 is in its P or dS pass meanwhile, so the tensor core
    // has work while each team computes. Each accumulator is summed in a
    // fixed order, so the sums are deterministic.
    constexpr bool kSplit = Sh::kIssuers == 2;
    const bool do_a = !kSplit || warp == 1;  // S^T and dV
    const bool do_b = !kSplit || warp == 2;  // dP^T and dK
    if (elect_one()) {
      constexpr uint32_t id_s = idesc_f16(kBF16, 128, Sh::kQRows, false, false);  // S^T, dP^T
      constexpr uint32_t id_dv = idesc_f16(kBF16, 128, kD, false, true);          // P^T (tmem) x dO
      constexpr uint32_t id_dk = idesc_f16(kBF16, 128, kD, false, true);          // dS^T (tmem) x Q
      const uint32_t sK = smem_u32(smem + Sh::kOffK);
      const uint32_t sV = smem_u32(smem + Sh::kOffV);
      bool ok = bwd_wait(&bars->kv_full, 0, abort, kSite + 2);
      tc_fence_after();
      auto kmajor_kv = [](uint32_t base, int kk) {
        return sdesc_sw128(base + (kk >> 2) * Sh::kChunkBytes + (kk & 3) * 32, 16, 1024);
      };
      auto kmajor_q = [](uint32_t base, int kk) {
        return sdesc_sw128(base + (kk >> 2) * Sh::kQChunkBytes + (kk & 3) * 32, 16, 1024);
      };
      auto mnmajor_q = [](uint32_t base, int kk) {
        return sdesc_sw128(base + kk * 2048, Sh::kQChunkBytes, 1024);
      };
      auto q_addr = [&](int it) {
        return smem_u32(smem + Sh::kOffQ + (it % Sh::kSlots) * 2 * Sh::kQTileBytes);
      };
      auto wait_q = [&](int it) {
        const bool r = bwd_wait(&bars->qd_full[it % Sh::kSlots],
                                static_cast<uint32_t>(it / Sh::kSlots) & 1u, abort, kSite + 3);
        tc_fence_after();
        return r;
      };
      auto issue_s = [&](int it) {  // S^T = K Q^T -> region A of the item's team
        const uint32_t sQ = q_addr(it);
        const uint32_t d = tmem + Sh::kColA + Sh::kQRows * (it & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_ss(d, kmajor_kv(sK, kk), kmajor_q(sQ, kk), id_s, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_ready[it & 1]);
      };
      auto issue_dp = [&](int it) {  // dP^T = V dO^T -> region B of the item's team
        const uint32_t sDO = q_addr(it) + Sh::kQTileBytes;
        const uint32_t d = tmem + Sh::kColB + Sh::kQRows * (it & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_ss(d, kmajor_kv(sV, kk), kmajor_q(sDO, kk), id_s, kk > 0 ? 1u : 0u);
        umma_commit(&bars->dp_ready[it & 1]);
      };
      for (int it = 0; it < 2 && it < n_items && ok; ++it) {
        if ((ok = wait_q(it))) {
          if (do_a) issue_s(it);
          if (kDoDK && do_b) issue_dp(it);
        }
      }
      for (int it = 0; it < n_items && ok; ++it) {
        const int t = it & 1;
        const uint32_t ph = static_cast<uint32_t>(it >> 1) & 1u;
        const uint32_t sQ = q_addr(it);
        const uint32_t sDO = sQ + Sh::kQTileBytes;
        const uint32_t acc_first = (it == 0) ? 0u : 1u;
        const bool more = it + 2 < n_items;
        if (do_a) {
          // the team's P pass of item it: P^T in region A (dV's operand), or,
          // in the dK pass, S^T read out of region A into registers
          if (!(ok = bwd_wait(&bars->p_ready[t], ph, abort, kSite + 4))) break;
          tc_fence_after();
          if constexpr (kDoDV) {
            // dV += P^T dO: A = P^T of the team's region (queries [32c, 32c+32)
            // packed into columns [32c, 32c+16), 16 queries = 8 columns per step)
#pragma unroll
            for (int kk = 0; kk < Sh::kQRows / 16; ++kk)
              umma_ts(tmem + Sh::kColDV, tmem + Sh::kColA + Sh::kQRows * t + (kk >> 1) * 32 + (kk & 1) * 8,
                      mnmajor_q(sDO, kk), id_dv, (kk == 0) ? acc_first : 1u);
          }
          if (more) {
            if (!(ok = wait_q(it + 2))) break;
            issue_s(it + 2);
          }
        }
        if (kDoDK && do_b) {
          // dK += dS^T Q: A = dS^T of the team's region B, packed like P^T
          if (!(ok = bwd_wait(&bars->ds_ready[t], ph, abort, kSite + 5))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < Sh::kQRows / 16; ++kk)
            umma_ts(tmem + Sh::kColDK, tmem + Sh::kColB + Sh::kQRows * t + (kk >> 1) * 32 + (kk & 1) * 8,
                    mnmajor_q(sQ, kk), id_dk, (kk == 0) ? acc_first : 1u);
        }
        // the slot is free once the readers of it that this thread issued
        // have run (each issuer commits once)
        umma_commit(&bars->qd_empty[it % Sh::kSlots]);
        if (kDoDK && do_b && more) {
          if (kSplit && !(ok = wait_q(it + 2))) break;
          issue_dp(it + 2);
        }
      }
      umma_commit(&bars->final_done);
      const int di = kSplit ? warp - 1 : 0;
      umma_commit(&bars->drain[di]);
      mbar_wait(&bars->drain[di], 0, kWaitTimeoutNs, kSite + 12);
    }
    __syncwarp();
  } else {
    // ======================= compute teams =======================
    const int team = (warp - Sh::kFirst) / (4 * Sh::kGroups);
    const int g = ((warp - Sh::kFirst) >> 2) % Sh::kGroups;  // group within the team
    const int lane_base = 32 * (warp & 3);
    const int r = lane_base + lane;             // key row within the tile
    const int key = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(lane_base) << 16;
    // this group's 32 query columns of the team's S^T / dP^T, and the 16
    // columns its P^T / dS^T (16-bit pairs) overwrite: only columns it has
    // read itself
    const uint32_t t_a = tmem + lane_off + Sh::kColA + Sh::kQRows * team + 32 * g;
    const uint32_t t_b = tmem + lane_off + Sh::kColB + Sh::kQRows * team + 32 * g;
    constexpr bool alibi = kAlibi;  // compiled in only where used
    bool ok = true;
    for (int it = team; it < n_items; it += 2) {
      const uint32_t ph = static_cast<uint32_t>(it >> 1) & 1u;
      const int q0 = (i_begin + it % i_cnt) * Sh::kQRows;
      const float sl2 = alibi_slope2(p, b, kvh * p.group + it / i_cnt);
      // the group's 32 query columns of -LSE and Drow, bulk-loaded with the
      // item's Q/dO into its slot (the slot is refilled only after dK of this
      // item, which waits for this team's dS pass)
      const int slot = it % Sh::kSlots;
      const float* glse = reinterpret_cast<const float*>(smem + Sh::kOffVec + slot * Sh::kVecBytes) + 32 * g;
      const float* gdrow = glse + Sh::kQRows;
      // w first holds the 32 columns' -LSE, loaded before S^T is ready
      // (shared-memory loads are slow while the tensor core reads its
      // operands), then P (* (1 - tanh^2)) for the dS pass
      float w[32];
      if (!(ok = bwd_wait(&bars->qd_full[slot], static_cast<uint32_t>(it / Sh::kSlots) & 1u, abort, kSite + 6))) break;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 l4 = *reinterpret_cast<const float4*>(glse + 4 * j4);
        w[4 * j4] = l4.x;
        w[4 * j4 + 1] = l4.y;
        w[4 * j4 + 2] = l4.z;
        w[4 * j4 + 3] = l4.w;
      }
      if (!(ok = bwd_wait(&bars->s_ready[team], ph, abort, kSite + 7))) break;
      tc_fence_after();
      // does any (key, query) of this warp's 32 keys x the group's 32 queries need masking?
      const int kw_lo = k0 + lane_base, kw_hi = kw_lo + 31;
      const int qg_lo = q0 + 32 * g, qg_hi = qg_lo + 31;
      bool need_mask = (kw_hi >= seq_len) || (qg_hi >= seq_len);
      if (p.wr >= 0) need_mask |= (kw_hi > qg_lo + p.wr);
      if (p.wl >= 0) need_mask |= (kw_lo < qg_hi - p.wl);
      // pass 1: P^T from S^T -> TMEM; keep w = P (* (1 - tanh^2) under
      // softcap) for the dS pass
      {
        uint32_t sr[32];
        tmem_ld32(t_a, sr);
        tmem_ld_wait();
        const bool poly = kCap ? poly_ok(sr, p.cap_in) : false;
        // exponents first (w holds -LSE per column), then every exponential
        // before any result is consumed, so they pipeline
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const float2 s2 = make_float2(__uint_as_float(sr[2 * j2]), __uint_as_float(sr[2 * j2 + 1]));
          float2 x, fac;
          bwd_logit2<kCap>(s2, poly, p, make_float2(w[2 * j2], w[2 * j2 + 1]), x, fac);
          w[2 * j2] = x.x;
          w[2 * j2 + 1] = x.y;
          if constexpr (kCap) {  // the raw scores are no longer needed
            sr[2 * j2] = __float_as_uint(fac.x);
            sr[2 * j2 + 1] = __float_as_uint(fac.y);
          }
        }
        if constexpr (alibi)  // -slope * |query - key| in the exp2 domain
          alibi32(w, sl2, static_cast<float>(qg_lo - key), 1.f, p.wr == 0);
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = ex2_approx(w[i]);
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int qi = qg_lo + i;
            bool v = key < seq_len && qi < seq_len;
            if (p.wr >= 0) v = v && key <= qi + p.wr;
            if (p.wl >= 0) v = v && key >= qi - p.wl;
            w[i] = v ? w[i] : 0.f;
          }
        }
        if constexpr (kDoDV) {
          uint32_t pk[16];
#pragma unroll
          for (int j2 = 0; j2 < 16; ++j2) pk[j2] = pack2_alu<kBF16>(w[2 * j2], w[2 * j2 + 1]);
          tmem_st16(t_a, pk);
        }
        if constexpr (kCap) {
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] *= __uint_as_float(sr[i]);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready[team]);  // dV may start (or S may be overwritten)
      if constexpr (!kDoDK) continue;
      // pass 2: dS^T = w * (dP^T - Drow) -> TMEM region B (the dK operand),
      // once dP^T is in TMEM (dK two items back, the last reader of these
      // columns, precedes the dP^T MMA in issue order)
      if (!(ok = bwd_wait(&bars->dp_ready[team], ph, abort, kSite + 8))) break;
      tc_fence_after();
      {
        uint32_t dr[32];
        tmem_ld32(t_b, dr);
        tmem_ld_wait();
        uint32_t dsk[16];
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const int jl = 4 * j4;
          float4 d4 = *reinterpret_cast<const float4*>(gdrow + jl);
          if (need_mask) {
            // rows past the sequence end: the slot holds stale values (w = 0)
            const int q4 = qg_lo + jl;
            d4.x = q4 < seq_len ? d4.x : 0.f;
            d4.y = q4 + 1 < seq_len ? d4.y : 0.f;
            d4.z = q4 + 2 < seq_len ? d4.z : 0.f;
            d4.w = q4 + 3 < seq_len ? d4.w : 0.f;
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int j2 = 2 * j4 + h2;
            const float2 dp2 = make_float2(__uint_as_float(dr[2 * j2]), __uint_as_float(dr[2 * j2 + 1]));
            const float2 d2 = h2 == 0 ? make_float2(-d4.x, -d4.y) : make_float2(-d4.z, -d4.w);
            const float2 ds = __fmul2_rn(__fadd2_rn(dp2, d2), make_float2(w[jl + 2 * h2], w[jl + 2 * h2 + 1]));
            dsk[j2] = pack2<kBF16>(ds.x, ds.y);  // one conversion a pair (no ex2 in this pass)
          }
        }
        tmem_st16(t_b, dsk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready[team]);
    }

    // ---- epilogue: compute group e (four warps from kFirst + 4e) writes
    // its share of the rows: both accumulators, groups 0-1 the two column
    // halves of dV and 2-3 those of dK; one accumulator, each of the
    // 2 kGroups groups its share of the row ----
    if (ok) ok = bwd_wait(&bars->final_done, 0, abort, kSite + 9);
    tc_fence_after();
    const int e = (warp - Sh::kFirst) >> 2;
    const bool is_dk = kPass == kDkdvBoth ? e >= 2 : kPass == kDkOnly;
    void* outp = is_dk ? p.dk : p.dv;
    const uint32_t col = is_dk ? Sh::kColDK : Sh::kColDV;
    const float osc = is_dk ? p.scale : 1.f;  // dK = scale * dS^T Q
    constexpr int kHalfChunks = kPass == kDkdvBoth ? kD / 64 : kD / 32 / (2 * Sh::kGroups);
    const int c_begin = (kPass == kDkdvBoth ? (e & 1) : e) * kHalfChunks;
    uint8_t* dst = static_cast<uint8_t*>(outp) +
                   (static_cast<size_t>(seq_start + key) * p.dkv_tok + static_cast<size_t>(kvh) * kD) * 2;
    if (ok && n_items > 0) {
      // every lane loads (the TMEM load is warp-collective); only rows of
      // the sequence are stored
#pragma unroll 1
      for (int c = c_begin; c < c_begin + kHalfChunks; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_off + col + c * 32, rr);
        tmem_ld_wait();
        uint32_t wv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wv[i] = pack2<kBF16>(__uint_as_float(rr[2 * i]) * osc, __uint_as_float(rr[2 * i + 1]) * osc);
        if (key < seq_len) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
        }
      }
    } else if (ok && key < seq_len) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + c_begin * 64);
      for (int i = 0; i < kHalfChunks * 4; ++i) d4[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::kTmemCols);
  }
}

// ===========================================================================
// dQ, D = 256 (bwd_dq256_kernel; D = 64 and 128 use bwd_dq_kernel below)
// ===========================================================================
// The template keeps the general form of this design (D <= 128 first used
// it); only D = 256 is instantiated.
// One CTA per (sequence, query head, 128-row Q tile). Q and dO stay in tensor
// memory as the A operands of S = Q K^T and dP = dO V^T, so shared memory
// carries only the streamed K/V blocks; an item is one 64-key block:
//   warp 0      TMA producer: K_j, V_j (64 rows each) into a ring of slots.
//   warp 1      MMA issuer: S_j -> S_t, dP_j -> dP_t (t = j % 2), then
//               dQ += dS_j K_j with dS_j read from S_t.
//   warps 2-17  two teams of two compute groups, one thread per query row;
//               team t takes the items with j % 2 == t, group g of a team the
//               item's key columns [32g, 32g+32): P = exp(S - LSE), then
//               dS = P * (dP - Drow) (16-bit pairs) over the first half of the
//               S columns it has read. LSE and Drow of the row live in
//               registers. At the start warps 2-9 write Q and dO into TMEM.
// TMEM columns: Q [0, D/2), dO [D/2, D), S_t [128+64t, +64), dP_t
// [256+64t, +64), dQ [384, 384+D).
// MMA order per item j (team t): dQ_j (after the dS pass of j), S_{j+2} -> S_t,
// dP_{j+2} -> dP_t. While one team computes, the tensor core runs the other
// team's products; the order is fixed, so dQ is deterministic.
//
// D = 256: Q (128 columns) and dQ (256) fill TMEM with S and dP, so dO stays
// in shared memory (loaded once by TMA, the A operand of dP = dO V^T), an
// item is 32 keys and each team has one compute group.
template <int kD>
struct Dq256Shape {
  static_assert(kD == 256, "D <= 128 takes bwd_dq_kernel");
  static constexpr int kChunks = kD / 64;
  static constexpr int kKRows = kD == 256 ? 32 : 64;   // keys per item
  static constexpr int kGroups = kKRows / 32;          // compute groups per team
  static constexpr bool kDOSmem = kD == 256;           // dO in shared memory
  static constexpr int kChunkBytes = kKRows * 128;     // kKRows rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  // K/V ring slots (one tile each): six items in flight hide the L2 -> shared
  // latency of the next blocks behind about 1.3k cycles per item
  static constexpr int kStages = kD == 256 ? 8 : (kD == 128 ? 12 : 24);
  static constexpr int kOffKV = 0;
  static constexpr int kOffDO = kOffKV + kStages * kTileBytes;     // D = 256: dO, 128 rows
  static constexpr int kDOBytes = kDOSmem ? kChunks * 128 * 128 : 0;
  static constexpr int kOffBar = kOffDO + kDOBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
  static constexpr int kThreads = 64 + 2 * kGroups * 128;
  static constexpr int kTmemCols = 512;
  static constexpr int kColQ = 0;
  static constexpr int kColDO = kD / 2;                // (D <= 128)
  static constexpr int kColS = 128;                    // + kKRows t
  static constexpr int kColDP = kDOSmem ? 128 + 2 * kKRows : 256;  // + kKRows t
  static constexpr int kColDQ = kDOSmem ? 256 : 384;
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB a CTA may use");
  static_assert(kStages <= 24, "more ring slots than the barrier block holds");
};

struct Dq256Bars {
  uint64_t qd_tmem;      // Q (and dO, D <= 128) written to TMEM (4 kGroups warps)
  uint64_t do_full;      // D = 256: the dO tile in shared memory
  uint64_t kv_full[24];
  uint64_t kv_empty[24];
  uint64_t s_ready[2];
  uint64_t dp_ready[2];
  uint64_t ds_ready[2];
  uint64_t final_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int kD, bool kBF16, bool kCap, bool kAlibi>
__global__ void __launch_bounds__(Dq256Shape<kD>::kThreads, 1)
    bwd_dq256_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using Sh = Dq256Shape<kD>;
  static_assert(sizeof(Dq256Bars) <= Sh::kBarBytes, "barrier block exceeds its reservation");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Dq256Bars* bars = reinterpret_cast<Dq256Bars*>(smem + Sh::kOffBar);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (sequence, head) major; Q tiles with most keys first
  const int nq = p.n_ktiles;  // 128-row tiles per sequence
  const int bh = static_cast<int>(blockIdx.x) / nq;
  const int qt = nq - 1 - static_cast<int>(blockIdx.x) % nq;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  int seq_start, seq_len;
  if (p.cu_seqlens != nullptr) {
    seq_start = p.cu_seqlens[b];
    seq_len = p.cu_seqlens[b + 1] - seq_start;
  } else {
    seq_start = b * p.S;
    seq_len = p.S;
  }
  const int q0 = qt * 128;
  if (q0 >= seq_len) return;
  const int kvh = h / p.group;
  const int row_hi = min(q0 + 127, seq_len - 1);
  int key_hi = seq_len - 1;
  if (p.wr >= 0) key_hi = min(key_hi, row_hi + p.wr);
  int key_lo = 0;
  if (p.wl >= 0) key_lo = max(0, q0 - p.wl);
  const int n_begin = key_lo / Sh::kKRows;
  const int n_tiles = key_hi >= key_lo ? key_hi / Sh::kKRows + 1 - n_begin : 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qd_tmem, 4 * Sh::kGroups);
    mbar_init(&bars->do_full, 1);
    for (int i = 0; i < Sh::kStages; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_ready[t], 1);
      mbar_init(&bars->dp_ready[t], 1);
      mbar_init(&bars->ds_ready[t], 4 * Sh::kGroups);
    }
    mbar_init(&bars->final_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, Sh::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (elect_one()) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if constexpr (Sh::kDOSmem) {
        mbar_arrive_expect_tx(&bars->do_full, Sh::kDOBytes);
        for (int c = 0; c < Sh::kChunks; ++c)
          tma_load_3d(&tm_do, &bars->do_full, smem + Sh::kOffDO + c * 128 * 128, c * 64, h,
                      seq_start + q0);
      }
      int fill = 0;
      for (int j = 0; j < n_tiles && !*abort; ++j) {
        const int tok = seq_start + (n_begin + j) * Sh::kKRows;
        for (int kv = 0; kv < 2; ++kv, ++fill) {
          const int slot = fill % Sh::kStages;
          const uint32_t ph = static_cast<uint32_t>(fill / Sh::kStages) & 1u;
          if (!bwd_wait(&bars->kv_empty[slot], ph ^ 1u, abort, 401)) break;
          mbar_arrive_expect_tx(&bars->kv_full[slot], Sh::kTileBytes);
          uint8_t* dst = smem + Sh::kOffKV + slot * Sh::kTileBytes;
          const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
          for (int c = 0; c < Sh::kChunks; ++c)
            tma_load_3d(tm, &bars->kv_full[slot], dst + c * Sh::kChunkBytes, c * 64, kvh, tok);
        }
      }
      for (int f = max(0, fill - Sh::kStages); f < fill; ++f)
        mbar_wait(&bars->kv_full[f % Sh::kStages], static_cast<uint32_t>(f / Sh::kStages) & 1u, kWaitTimeoutNs, 409);
      if constexpr (Sh::kDOSmem) mbar_wait(&bars->do_full, 0, kWaitTimeoutNs, 410);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (elect_one()) {
      constexpr uint32_t id_s = idesc_f16(kBF16, 128, Sh::kKRows, false, false);  // S, dP
      constexpr uint32_t id_dq = idesc_f16(kBF16, 128, kD, false, true);          // dS (tmem) x K
      const uint32_t sKV = smem_u32(smem + Sh::kOffKV);
      const uint32_t sDO = smem_u32(smem + Sh::kOffDO);
      bool ok = bwd_wait(&bars->qd_tmem, 0, abort, 402);
      if (ok && Sh::kDOSmem) ok = bwd_wait(&bars->do_full, 0, abort, 403);
      tc_fence_after();
      auto kmajor = [](uint32_t base, int kk) {
        return sdesc_sw128(base + (kk >> 2) * Sh::kChunkBytes + (kk & 3) * 32, 16, 1024);
      };
      auto wait_slot = [&](int fill) {
        const bool r = bwd_wait(&bars->kv_full[fill % Sh::kStages],
                                static_cast<uint32_t>(fill / Sh::kStages) & 1u, abort, 404);
        tc_fence_after();
        return r;
      };
      auto slot_addr = [&](int fill) { return sKV + (fill % Sh::kStages) * Sh::kTileBytes; };
      auto issue_s = [&](int j) {  // S_j = Q K_j^T -> S_{j%2}
        const uint32_t sK = slot_addr(2 * j);
        const uint32_t d = tmem + Sh::kColS + Sh::kKRows * (j & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_ts(d, tmem + Sh::kColQ + 8 * kk, kmajor(sK, kk), id_s, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_ready[j & 1]);
      };
      auto issue_dp = [&](int j) {  // dP_j = dO V_j^T -> dP_{j%2}
        const uint32_t sV = slot_addr(2 * j + 1);
        const uint32_t d = tmem + Sh::kColDP + Sh::kKRows * (j & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          if constexpr (Sh::kDOSmem)  // A = the dO tile, K-major, 128-row chunks
            umma_ss(d, sdesc_sw128(sDO + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024),
                    kmajor(sV, kk), id_s, kk > 0 ? 1u : 0u);
          else
            umma_ts(d, tmem + Sh::kColDO + 8 * kk, kmajor(sV, kk), id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->dp_ready[j & 1]);
      };
      for (int j = 0; j < 2 && j < n_tiles && ok; ++j) {
        if (!(ok = wait_slot(2 * j))) break;
        issue_s(j);
        if (!(ok = wait_slot(2 * j + 1))) break;
        issue_dp(j);
      }
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int t = j & 1;
        if (!(ok = bwd_wait(&bars->ds_ready[t], static_cast<uint32_t>(j >> 1) & 1u, abort, 405))) break;
        tc_fence_after();
        // dQ += dS_j K_j: A = dS_j from S_t (keys [32c, 32c+32) packed into
        // columns [32c, 32c+16)), B = K_j with N = D (MN-major)
        {
          const uint32_t sK = slot_addr(2 * j);
          const uint32_t a = tmem + Sh::kColS + Sh::kKRows * t;
#pragma unroll
          for (int kk = 0; kk < Sh::kKRows / 16; ++kk)
            umma_ts(tmem + Sh::kColDQ, a + (kk >> 1) * 32 + (kk & 1) * 8,
                    sdesc_sw128(sK + kk * 2048, Sh::kChunkBytes, 1024), id_dq,
                    (j == 0 && kk == 0) ? 0u : 1u);
        }
        umma_commit(&bars->kv_empty[(2 * j) % Sh::kStages]);      // K_j
        umma_commit(&bars->kv_empty[(2 * j + 1) % Sh::kStages]);  // V_j
        // S_{j+2} and dP_{j+2}: dQ_j, the last reader of S_t, precedes them;
        // the team read dP_t before signalling ds_ready
        if (j + 2 < n_tiles) {
          if (!(ok = wait_slot(2 * (j + 2)))) break;
          issue_s(j + 2);
          if (!(ok = wait_slot(2 * (j + 2) + 1))) break;
          issue_dp(j + 2);
        }
      }
      umma_commit(&bars->final_done);
      umma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, kWaitTimeoutNs, 411);
    }
    __syncwarp();
  } else {
    // ======================= compute teams =======================
    const int team = (warp - 2) / (4 * Sh::kGroups);
    const int g = ((warp - 2) >> 2) % Sh::kGroups;  // group within the team
    const int lane_base = 32 * (warp & 3);
    const int r = lane_base + lane;          // query row within the tile
    const int qrow = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(lane_base) << 16;
    if (team == 0) {  // (D = 256: group 0 only, Q; dO arrives by TMA)
      // Q (group 0) or dO (group 1) row -> TMEM, two 16-bit values per column
      // (the A-operand layout: K-step kk of 16 values at columns 8kk..8kk+7);
      // rows past the sequence end are zero
      const uint16_t* src = g == 0 ? static_cast<const uint16_t*>(p.q) +
                                         static_cast<size_t>(seq_start + qrow) * p.q_tok + static_cast<size_t>(h) * kD
                                   : static_cast<const uint16_t*>(p.dout) +
                                         (static_cast<size_t>(seq_start + qrow) * p.Hq + h) * kD;
      const uint32_t col = g == 0 ? Sh::kColQ : Sh::kColDO;
#pragma unroll
      for (int c = 0; c < kD / 64; ++c) {
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint4 u = make_uint4(0u, 0u, 0u, 0u);
          if (qrow < seq_len) u = reinterpret_cast<const uint4*>(src + c * 64)[i];
          v[4 * i] = u.x;
          v[4 * i + 1] = u.y;
          v[4 * i + 2] = u.z;
          v[4 * i + 3] = u.w;
        }
        tmem_st32(tmem + lane_off + col + 32 * c, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->qd_tmem);
    }
    // the row's -LSE (exp2 domain) and Drow
    float nlse = -INFINITY, drow = 0.f;
    if (qrow < seq_len) {
      const size_t vi = vec_index(p, h, b, seq_start, qrow);
      nlse = p.vec_nlse[vi];
      drow = p.vec_drow[vi];
    }
    const float2 nl2 = make_float2(nlse, nlse);
    const float2 nd2 = make_float2(-drow, -drow);
    constexpr bool alibi = kAlibi;  // compiled in only where used
    const float sl2 = alibi_slope2(p, b, h);
    bool ok = true;
    for (int j = team; j < n_tiles; j += 2) {
      const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
      if (!(ok = bwd_wait(&bars->s_ready[team], ph, abort, 406))) break;
      tc_fence_after();
      const int k0 = (n_begin + j) * Sh::kKRows + 32 * g;  // first key of this group's columns
      const uint32_t t_s = tmem + lane_off + Sh::kColS + Sh::kKRows * team + 32 * g;
      const uint32_t t_dp = tmem + lane_off + Sh::kColDP + Sh::kKRows * team + 32 * g;
      // mask needed for this warp's 32 rows x the group's 32 keys?
      const int r_lo = q0 + lane_base, r_hi = r_lo + 31;
      bool need_mask = (k0 + 31 >= seq_len) || (r_hi >= seq_len);
      if (p.wr >= 0) need_mask |= (k0 + 31 > r_lo + p.wr);
      if (p.wl >= 0) need_mask |= (k0 < r_hi - p.wl);
      // pass 1 (needs S_j only): w = P (* (1 - tanh^2)) for the group's 32
      // keys, kept in registers
      float w[32];
      {
        uint32_t sr[32];
        tmem_ld32(t_s, sr);
        tmem_ld_wait();
        bwd_probs32<kCap>(sr, nl2, p, alibi, sl2, static_cast<float>(qrow - k0), w, p.wr == 0);
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kj = k0 + i;
            bool v = qrow < seq_len && kj < seq_len;
            if (p.wr >= 0) v = v && kj <= qrow + p.wr;
            if (p.wl >= 0) v = v && kj >= qrow - p.wl;
            w[i] = v ? w[i] : 0.f;
          }
        }
      }
      // pass 2 (needs dP_j): dS = w * (dP - Drow) -> the S columns already read
      if (!(ok = bwd_wait(&bars->dp_ready[team], ph, abort, 407))) break;
      tc_fence_after();
      {
        uint32_t dr[32];
        tmem_ld32(t_dp, dr);
        tmem_ld_wait();
        uint32_t dsk[16];
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const float2 dp2 = make_float2(__uint_as_float(dr[2 * j2]), __uint_as_float(dr[2 * j2 + 1]));
          const float2 ds = __fmul2_rn(__fadd2_rn(dp2, nd2), make_float2(w[2 * j2], w[2 * j2 + 1]));
          dsk[j2] = pack2<kBF16>(ds.x, ds.y);  // one conversion a pair (no ex2 in this pass)
        }
        // dS of keys [k0, k0 + 32) -> columns [32g, 32g + 16) of S_t
        // (columns this group has already read)
        tmem_st16(t_s, dsk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready[team]);
    }
    // ---- epilogue: dQ row -> dq; the 2 kGroups warp groups write the
    // 32-column chunks e * kPer .. (e + 1) * kPer - 1 of their rows (D = 64:
    // groups 2, 3 have none) ----
    if (ok) ok = bwd_wait(&bars->final_done, 0, abort, 408);
    tc_fence_after();
    const int e = (warp - 2) >> 2;
    constexpr int kPer = (kD / 32 + 2 * Sh::kGroups - 1) / (2 * Sh::kGroups);
    uint8_t* dst = static_cast<uint8_t*>(p.dq) +
                   (static_cast<size_t>(seq_start + qrow) * p.dq_tok + static_cast<size_t>(h) * kD) * 2;
#pragma unroll 1
    for (int c = e * kPer; c < (e + 1) * kPer && c < kD / 32; ++c) {
      if (ok && n_tiles > 0) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_off + Sh::kColDQ + c * 32, rr);
        tmem_ld_wait();
        uint32_t wv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wv[i] = pack2<kBF16>(__uint_as_float(rr[2 * i]) * p.scale, __uint_as_float(rr[2 * i + 1]) * p.scale);
        if (qrow < seq_len) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
        }
      } else if (ok && qrow < seq_len) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 64);
        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::kTmemCols);
  }
}

// ===========================================================================
// dQ (D = 64, 128)
// ===========================================================================
// One CTA per (sequence, query head, 128-row Q tile); an item is one 128-key
// block, so every product has N = 128 (N = D for dQ += dS K):
//   warp 0      TMA producer: the Q and dO tiles once, then K_j and V_j
//               (128 rows each) into two rings: V_j is free once dP_j has
//               run, K_j only after dQ_j.
//   warp 1      MMA issuer and TMEM owner.
//   warps 2-17  four compute groups of four warps, one thread per query row;
//               group g takes the key columns [32g, 32g + 32) of each block:
//               P = exp(S - LSE) into registers, then dS = P * (dP - Drow)
//               (16-bit pairs) over the first half of the dP columns it has
//               read.
// TMEM columns: S [0, 128), dP_t [128 + 128t, +128) for t = j % 2, dQ
// [384, 384 + D). Q and dO stay in shared memory as the A operands of
// S = Q K^T and dP = dO V^T, which leaves tensor memory room for two dP
// buffers: the P pass frees S as soon as it has read it, and dP_{j+1} needs
// only dQ_{j-1} (the last reader of its buffer) to be issued, so S_{j+1} and
// dP_{j+1} run while the groups form P_j and dS_j. MMA order: S_{j+1},
// dP_{j+1}, dQ_j; the order is fixed, so dQ is deterministic.
template <int kD>
struct DqShape {
  static_assert(kD == 64 || kD == 128, "this dQ kernel takes D = 64 or 128");
  static constexpr int kChunks = kD / 64;
  static constexpr int kKRows = 128;                   // keys per item
  static constexpr int kGroups = 4;                    // 32 key columns each
  static constexpr int kChunkBytes = 128 * 128;        // 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTileBytes;
  static constexpr int kKStages = kD == 128 ? 3 : 6;   // K ring slots
  static constexpr int kVStages = kD == 128 ? 2 : 4;   // V ring slots
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
  static constexpr int kThreads = 64 + kGroups * 128;
  static constexpr int kTmemCols = 512;
  static constexpr int kColS = 0;
  static constexpr int kColDP = 128;                   // + 128 t
  static constexpr int kColDQ = 384;
  static constexpr int kPolyOf8 = 2;  // FMA-pipe share of the exponentials
  static_assert(kSmemBytes <= 232448, "shared memory exceeds the 227 KB a CTA may use");
  static_assert(kKStages <= 8 && kVStages <= 8, "more ring slots than the barrier block holds");
};

struct DqBars {
  uint64_t qdo_full;     // the Q and dO tiles
  uint64_t k_full[8];
  uint64_t k_empty[8];
  uint64_t v_full[8];
  uint64_t v_empty[8];
  uint64_t s_ready;
  uint64_t s_free;       // every group has read S
  uint64_t dp_ready[2];  // per dP buffer
  uint64_t ds_ready[2];
  uint64_t final_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int kD, bool kBF16, bool kCap, bool kAlibi>
__global__ void __launch_bounds__(DqShape<kD>::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using Sh = DqShape<kD>;
  static_assert(sizeof(DqBars) <= Sh::kBarBytes, "barrier block exceeds its reservation");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DqBars* bars = reinterpret_cast<DqBars*>(smem + Sh::kOffBar);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (sequence, head) major; Q tiles with most keys first
  const int nq = p.n_ktiles;  // 128-row tiles per sequence
  const int bh = static_cast<int>(blockIdx.x) / nq;
  const int qt = nq - 1 - static_cast<int>(blockIdx.x) % nq;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  int seq_start, seq_len;
  if (p.cu_seqlens != nullptr) {
    seq_start = p.cu_seqlens[b];
    seq_len = p.cu_seqlens[b + 1] - seq_start;
  } else {
    seq_start = b * p.S;
    seq_len = p.S;
  }
  const int q0 = qt * 128;
  if (q0 >= seq_len) return;
  const int kvh = h / p.group;
  const int row_hi = min(q0 + 127, seq_len - 1);
  int key_hi = seq_len - 1;
  if (p.wr >= 0) key_hi = min(key_hi, row_hi + p.wr);
  int key_lo = 0;
  if (p.wl >= 0) key_lo = max(0, q0 - p.wl);
  const int n_begin = key_lo / Sh::kKRows;
  const int n_tiles = key_hi >= key_lo ? key_hi / Sh::kKRows + 1 - n_begin : 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qdo_full, 1);
    for (int i = 0; i < Sh::kKStages; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < Sh::kVStages; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    mbar_init(&bars->s_ready, 1);
    mbar_init(&bars->s_free, 4 * Sh::kGroups);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->dp_ready[t], 1);
      mbar_init(&bars->ds_ready[t], 4 * Sh::kGroups);
    }
    mbar_init(&bars->final_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, Sh::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      // (rows past the end of the tensor read as zero; rows of the next
      // sequence are masked out of P)
      mbar_arrive_expect_tx(&bars->qdo_full, 2 * Sh::kTileBytes);
      for (int c = 0; c < Sh::kChunks; ++c) {
        tma_load_3d(&tm_q, &bars->qdo_full, smem + Sh::kOffQ + c * Sh::kChunkBytes, c * 64, h, seq_start + q0);
        tma_load_3d(&tm_do, &bars->qdo_full, smem + Sh::kOffDO + c * Sh::kChunkBytes, c * 64, h, seq_start + q0);
      }
      int nk = 0, nv = 0;  // K and V tiles issued
      while (nv < n_tiles && !*abort) {
        const int tok = seq_start + (n_begin + nv) * Sh::kKRows;
        if (nk == nv) {
          const int slot = nk % Sh::kKStages;
          if (!bwd_wait(&bars->k_empty[slot], (static_cast<uint32_t>(nk / Sh::kKStages) & 1u) ^ 1u, abort, 401)) break;
          mbar_arrive_expect_tx(&bars->k_full[slot], Sh::kTileBytes);
          for (int c = 0; c < Sh::kChunks; ++c)
            tma_load_3d(&tm_k, &bars->k_full[slot], smem + Sh::kOffK + slot * Sh::kTileBytes + c * Sh::kChunkBytes,
                        c * 64, kvh, tok);
          ++nk;
        }
        const int slot = nv % Sh::kVStages;
        if (!bwd_wait(&bars->v_empty[slot], (static_cast<uint32_t>(nv / Sh::kVStages) & 1u) ^ 1u, abort, 409)) break;
        mbar_arrive_expect_tx(&bars->v_full[slot], Sh::kTileBytes);
        for (int c = 0; c < Sh::kChunks; ++c)
          tma_load_3d(&tm_v, &bars->v_full[slot], smem + Sh::kOffV + slot * Sh::kTileBytes + c * Sh::kChunkBytes,
                      c * 64, kvh, tok);
        ++nv;
      }
      // the copies still in flight finish before the CTA may exit
      for (int f = max(0, nk - Sh::kKStages); f < nk; ++f)
        mbar_wait(&bars->k_full[f % Sh::kKStages], static_cast<uint32_t>(f / Sh::kKStages) & 1u, kWaitTimeoutNs, 410);
      for (int f = max(0, nv - Sh::kVStages); f < nv; ++f)
        mbar_wait(&bars->v_full[f % Sh::kVStages], static_cast<uint32_t>(f / Sh::kVStages) & 1u, kWaitTimeoutNs, 410);
      mbar_wait(&bars->qdo_full, 0, kWaitTimeoutNs, 410);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (elect_one()) {
      constexpr uint32_t id_s = idesc_f16(kBF16, 128, Sh::kKRows, false, false);  // S, dP
      constexpr uint32_t id_dq = idesc_f16(kBF16, 128, kD, false, true);          // dS (tmem) x K
      const uint32_t sQ = smem_u32(smem + Sh::kOffQ);
      const uint32_t sDO = smem_u32(smem + Sh::kOffDO);
      const uint32_t sK0 = smem_u32(smem + Sh::kOffK);
      const uint32_t sV0 = smem_u32(smem + Sh::kOffV);
      bool ok = bwd_wait(&bars->qdo_full, 0, abort, 402);
      tc_fence_after();
      // 128 rows, K-major, 64-element chunks
      auto kmajor = [](uint32_t base, int kk) {
        return sdesc_sw128(base + (kk >> 2) * Sh::kChunkBytes + (kk & 3) * 32, 16, 1024);
      };
      auto k_addr = [&](int j) { return sK0 + (j % Sh::kKStages) * Sh::kTileBytes; };
      auto issue_s = [&](int j) {  // S_j = Q K_j^T
        if (!bwd_wait(&bars->k_full[j % Sh::kKStages], static_cast<uint32_t>(j / Sh::kKStages) & 1u, abort, 404))
          return false;
        tc_fence_after();
        const uint32_t sK = k_addr(j);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_ss(tmem + Sh::kColS, kmajor(sQ, kk), kmajor(sK, kk), id_s, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_ready);
        return true;
      };
      auto issue_dp = [&](int j) {  // dP_j = dO V_j^T -> buffer j % 2; V_j is then free
        if (!bwd_wait(&bars->v_full[j % Sh::kVStages], static_cast<uint32_t>(j / Sh::kVStages) & 1u, abort, 412))
          return false;
        tc_fence_after();
        const uint32_t sV = sV0 + (j % Sh::kVStages) * Sh::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_ss(tmem + Sh::kColDP + 128 * (j & 1), kmajor(sDO, kk), kmajor(sV, kk), id_s, kk > 0 ? 1u : 0u);
        umma_commit(&bars->dp_ready[j & 1]);
        umma_commit(&bars->v_empty[j % Sh::kVStages]);
        return true;
      };
      if (ok && n_tiles > 0) ok = issue_s(0) && issue_dp(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        const bool more = j + 1 < n_tiles;
        // S_{j+1} once every group has read S_j; dP_{j+1} into the buffer
        // that dQ_{j-1}, issued before, read
        if (!(ok = bwd_wait(&bars->s_free, static_cast<uint32_t>(j) & 1u, abort, 403))) break;
        if (more && !(ok = issue_s(j + 1) && issue_dp(j + 1))) break;
        // dQ += dS_j K_j: A = dS_j over dP buffer j % 2 (keys [32c, 32c + 32)
        // packed into columns [32c, 32c + 16)), B = K_j with N = D (MN-major)
        if (!(ok = bwd_wait(&bars->ds_ready[j & 1], static_cast<uint32_t>(j >> 1) & 1u, abort, 405))) break;
        tc_fence_after();
        const uint32_t sK = k_addr(j);
        const uint32_t a = tmem + Sh::kColDP + 128 * (j & 1);
#pragma unroll
        for (int kk = 0; kk < Sh::kKRows / 16; ++kk)
          umma_ts(tmem + Sh::kColDQ, a + (kk >> 1) * 32 + (kk & 1) * 8,
                  sdesc_sw128(sK + kk * 2048, Sh::kChunkBytes, 1024), id_dq, (j == 0 && kk == 0) ? 0u : 1u);
        umma_commit(&bars->k_empty[j % Sh::kKStages]);
      }
      umma_commit(&bars->final_done);
      umma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, kWaitTimeoutNs, 411);
    }
    __syncwarp();
  } else {
    // ======================= compute groups =======================
    const int g = (warp - 2) >> 2;           // key columns [32g, 32g + 32)
    const int lane_base = 32 * (warp & 3);
    const int r = lane_base + lane;          // query row within the tile
    const int qrow = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(lane_base) << 16;
    // the row's -LSE (exp2 domain) and Drow
    float nlse = -INFINITY, drow = 0.f;
    if (qrow < seq_len) {
      const size_t vi = vec_index(p, h, b, seq_start, qrow);
      nlse = p.vec_nlse[vi];
      drow = p.vec_drow[vi];
    }
    const float2 nl2 = make_float2(nlse, nlse);
    const float2 nd2 = make_float2(-drow, -drow);
    constexpr bool alibi = kAlibi;  // compiled in only where used
    const float sl2 = alibi_slope2(p, b, h);
    const uint32_t t_s = tmem + lane_off + Sh::kColS + 32 * g;
    const int r_lo = q0 + lane_base, r_hi = r_lo + 31;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (!(ok = bwd_wait(&bars->s_ready, static_cast<uint32_t>(j) & 1u, abort, 406))) break;
      tc_fence_after();
      const int k0 = (n_begin + j) * Sh::kKRows + 32 * g;  // first key of this group's columns
      // mask needed for this warp's 32 rows x the group's 32 keys?
      bool need_mask = (k0 + 31 >= seq_len) || (r_hi >= seq_len);
      if (p.wr >= 0) need_mask |= (k0 + 31 > r_lo + p.wr);
      if (p.wl >= 0) need_mask |= (k0 < r_hi - p.wl);
      // P pass (needs S_j only): w = P (* (1 - tanh^2)) for the group's 32
      // keys, kept in registers; S is free once every group has read it
      float w[32];
      {
        uint32_t sr[32];
        tmem_ld32(t_s, sr);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
        bwd_probs32<kCap, Sh::kPolyOf8>(sr, nl2, p, alibi, sl2, static_cast<float>(qrow - k0), w, p.wr == 0);
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kj = k0 + i;
            bool v = qrow < seq_len && kj < seq_len;
            if (p.wr >= 0) v = v && kj <= qrow + p.wr;
            if (p.wl >= 0) v = v && kj >= qrow - p.wl;
            w[i] = v ? w[i] : 0.f;
          }
        }
      }
      // dS pass (needs dP_j): dS = w * (dP - Drow) -> the dP columns already read
      if (!(ok = bwd_wait(&bars->dp_ready[j & 1], static_cast<uint32_t>(j >> 1) & 1u, abort, 407))) break;
      tc_fence_after();
      {
        const uint32_t t_dp = tmem + lane_off + Sh::kColDP + 128 * (j & 1) + 32 * g;
        uint32_t dr[32];
        tmem_ld32(t_dp, dr);
        tmem_ld_wait();
        uint32_t dsk[16];
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const float2 dp2 = make_float2(__uint_as_float(dr[2 * j2]), __uint_as_float(dr[2 * j2 + 1]));
          const float2 ds = __fmul2_rn(__fadd2_rn(dp2, nd2), make_float2(w[2 * j2], w[2 * j2 + 1]));
          dsk[j2] = pack2<kBF16>(ds.x, ds.y);  // one conversion a pair (no ex2 in this pass)
        }
        // dS of keys [k0, k0 + 32) -> columns [32g, 32g + 16) of the buffer
        tmem_st16(t_dp, dsk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready[j & 1]);
    }
    // ---- epilogue: dQ row -> dq; group g writes the 32-column chunk g of
    // its rows (D = 64: groups 0, 1) ----
    if (ok) ok = bwd_wait(&bars->final_done, 0, abort, 408);
    tc_fence_after();
    uint8_t* dst = static_cast<uint8_t*>(p.dq) +
                   (static_cast<size_t>(seq_start + qrow) * p.dq_tok + static_cast<size_t>(h) * kD) * 2;
    const int c = g;
    if (c < kD / 32) {
      if (ok && n_tiles > 0) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_off + Sh::kColDQ + c * 32, rr);
        tmem_ld_wait();
        uint32_t wv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wv[i] = pack2<kBF16>(__uint_as_float(rr[2 * i]) * p.scale, __uint_as_float(rr[2 * i + 1]) * p.scale);
        if (qrow < seq_len) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
        }
      } else if (ok && qrow < seq_len) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 64);
        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::kTmemCols);
  }
}

}  // namespace fa
