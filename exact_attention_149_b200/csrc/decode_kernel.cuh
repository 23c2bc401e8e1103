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

// grid B * Sq (one block per new token), block 128: 16 bytes per thread-step
template <bool kBF16>
__global__ void kv_append_kernel(const DecodeParams p) {
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
  uint16_t* kc = static_cast<uint16_t*>(p.k_cache) + dst;
  uint16_t* vc = static_cast<uint16_t*>(p.v_cache) + dst;
  for (int i = threadIdx.x; i < p.Hkv * groups; i += blockDim.x) {
    const int h = i / groups, d0 = (i % groups) * 8;
    const int e = h * p.D + d0;
    *reinterpret_cast<uint4*>(kc + e) = rotate8<kBF16>(kn + h * p.D, d0, cs, sn, p);
    *reinterpret_cast<uint4*>(vc + e) = *reinterpret_cast<const uint4*>(vn + e);
  }
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

// address of the 16-byte group `g` (0..7 within a 128-byte row) of row `r`
// of a TMA tile written with the 128-byte swizzle (tile base 1024-aligned)
__device__ __forceinline__ uint32_t sw128(uint32_t base, int r, int g) {
  return base + r * 128 + ((g ^ (r & 7)) << 4);
}

template <int kD>
struct DecShape {
  static constexpr int kTok = 64;                      // tokens per chunk
  static constexpr int kChunks = kD / 64;              // 128-byte column chunks
  static constexpr int kBoxBytes = kTok * 128;         // 64 rows x 128 B
  static constexpr int kKVBytes = kChunks * kBoxBytes; // K or V of one chunk
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kStages = kD == 128 ? 3 : 6;   // 2 CTAs per SM
  static constexpr int kBarOffset = kStages * kStageBytes;
  // cross-warp reduction scratch aliases the stage ring: it is written only
  // after every issued chunk has been consumed
  static constexpr int kRedOffset = 0;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;
  static constexpr int kThreads = 160;                 // 4 consumer warps + 1 producer
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
template <int kD, bool kBF16, int kNT>
__global__ void __launch_bounds__(160)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using Sh = DecShape<kD>;
  static_assert(sizeof(DecBars) <= 256, "barrier block exceeds its reservation");
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
        mbar_arrive_expect_tx(&bars->full[slot], Sh::kStageBytes);
        uint8_t* dst = smem + slot * Sh::kStageBytes;
        for (int c = 0; c < Sh::kChunks; ++c) {
          tma_load_3d(&tm_k, &bars->full[slot], dst + c * Sh::kBoxBytes, c * 64, kvh, row);
          tma_load_3d(&tm_v, &bars->full[slot], dst + Sh::kKVBytes + c * Sh::kBoxBytes, c * 64, kvh,
                      row);
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
  {
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
    const uint32_t kbase = sbase + slot * Sh::kStageBytes;
    const uint32_t vbase = kbase + Sh::kKVBytes;
    const int tok0 = warp * 16;  // this warp's 16 tokens of the chunk
    // ---- S^T = K Q^T ----
    float s[kNT][4];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      const int mi = lane >> 3, r = lane & 7;
      const int tok = tok0 + (mi & 1) * 8 + r;
      const int c = kk >> 2;
      const int g = (kk & 3) * 2 + (mi >> 1);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sw128(kbase + c * Sh::kBoxBytes, tok, g), a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) mma16816<kBF16>(s[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
    }
    // ---- logits, mask, online softmax ----
    const int wtok = (t_begin + i) * Sh::kTok + tok0;  // first token of this warp's 16
    const int pos0 = wtok + (lane >> 2);                // token of s[.][0], s[.][1]
    // every column sees all 16 tokens: no mask (warp-uniform)
    const bool all_visible = wtok >= lo_in && wtok + 16 <= hi_in;
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
#pragma unroll
      for (int mt = 0; mt < kD / 16; ++mt) {
        acc[nt][mt][0] *= al0;
        acc[nt][mt][1] *= al1;
        acc[nt][mt][2] *= al0;
        acc[nt][mt][3] *= al1;
      }
      // P^T fragments: transpose the two 8x8 blocks of the 16x8 accumulator
      pb[nt][0] = movmatrix_t(pack2<kBF16>(e0, e1));
      pb[nt][1] = movmatrix_t(pack2<kBF16>(e2, e3));
    }
    // ---- O^T += V^T P^T ----
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
      ldsm_x4_t(sw128(vbase + (dcol >> 6) * Sh::kBoxBytes, tok, (dcol & 63) >> 3), a0, a1, a2, a3);
      if (tail) {
        a0 &= vm01;
        a1 &= vm01;
        a2 &= vm23;
        a3 &= vm23;
      }
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) mma16816<kBF16>(acc[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->empty[slot]);
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
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt) {
      const int d0 = mt * 16 + (lane >> 2);
      red_o[(warp * kH + h0) * kD + d0] = acc[nt][mt][0];
      red_o[(warp * kH + h0 + 1) * kD + d0] = acc[nt][mt][1];
      red_o[(warp * kH + h0) * kD + d0 + 8] = acc[nt][mt][2];
      red_o[(warp * kH + h0 + 1) * kD + d0 + 8] = acc[nt][mt][3];
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
