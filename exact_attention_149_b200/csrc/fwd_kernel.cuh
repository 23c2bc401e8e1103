// Forward attention kernel for sm_100a.
//
// One CTA computes 256 query rows (two 128-row Q tiles) of one (sequence,
// query head) against the K/V tiles the mask leaves visible, with an online
// softmax ("FlashAttention 实战指南" §长序列注意力为什么会爆内存: tile Q, K,
// V into on-chip memory, update the row max and row sum tile by tile, never
// materialise the attention matrix).
//
// Warp roles (384 threads, three warpgroups):
//   warp 0      TMA producer: Q tiles once, then K_j, V_j into a ring of
//               shared-memory slots (128-byte swizzle).
//   warp 1      MMA issuer (one lane): S_t = Q_t K_j^T into TMEM, then
//               O_t += P_t V_j with P_t read from TMEM. Owns TMEM alloc.
//   warps 2-3   idle (they complete warpgroup 0, which gives its registers
//               to the softmax groups: 88 per thread instead of 168)
//   warps 4-7   softmax group 0 (Q tile 0), one thread per query row, 208
//               registers per thread (the whole score row lives in registers).
//   warps 8-11  softmax group 1 (Q tile 1).
// Register pool: 384 x 168 at launch = 64512 = 128 x 88 + 256 x 208.
// The two softmax groups alternate with the tensor core: while group 0
// exponentiates S_0, the tensor core runs group 1's PV and QK, and so on.
// Each group writes P_t in four 32-key parts and signals each one, so the
// tensor core starts PV_t on the first part while the rest of the row is
// still being exponentiated; a quarter of the exponentials are a cubic on
// the FMA pipe (ex2_poly2) so the special-function unit is not the only
// producer of P.
//
// TMEM columns (512 allocated): S_0 [0,128), S_1 [128,256), O_0 at 256,
// O_1 at 256 + D. P_t (16-bit, two per 32-bit column) overwrites the upper
// 64 columns of S_t after the row has been read into registers.
//
// The running max is only moved (and O rescaled) when a row max grows by
// more than 2^8 in the exp2 domain; otherwise the stale max is kept, which
// is exact after the final division by the row sum and keeps P <= 256.
#pragma once

#include "ptx.cuh"

namespace fa {

struct FwdParams {
  int B, Hq, Hkv, S, total;  // S: sequence length (max length when varlen)
  int group;                 // Hq / Hkv
  int n_qblocks;             // ceil(S / 256)
  int seq_blocks;            // varlen, B <= 64: blocks numbered sequence by sequence
  float scale_log2;          // scale * log2(e)
  float softcap;             // 0 = off
  float cap_in;              // scale / softcap
  float cap_out_log2;        // softcap * log2(e)
  int wl, wr;                // window, -1 = unbounded (causal already folded into wr)
  void* o;
  float* lse;
  const int* cu_seqlens;     // nullable
  const float* alibi;        // ALiBi slopes, nullable: slope of (b, h) = alibi[b * alibi_bstride + h]
  int alibi_bstride;
  float o_scale;             // FP8 inputs: the output's factor (v descale); unused otherwise
  unsigned long long wait_ns;  // limit of every bounded wait (4 s; shorter in the failure test)
};

// D = 256: one Q tile per CTA (S 128 + O 256 TMEM columns; two tiles would
// need 768) and one softmax warpgroup; Q (64 KB) and a two-slot K/V ring
// (64 KB a tile) fill shared memory.
//
// kF8: Q, K, V are FP8 E4M3 (one byte per element; the guide's §版本怎么选
// names an FP8 forward). A 128-byte swizzle row then holds 128 elements, a
// QK^T K-step is 32 elements (still 32 bytes), a PV K-step 32 keys, and P
// goes to the tensor core as E4M3, four per TMEM column. P is formed as
// 2^(x - m + kPOff) with the row's running max m moved whenever the true max
// exceeds it by more than kLazy, so the largest P of a row lies in
// [2^kPOff, 2^(kPOff + kLazy)] = [16, 256]: inside E4M3's range (448), with
// its 3-bit relative precision down to 2^-10 of the row's largest value.
template <int kD, bool kF8 = false>
struct FwdShape {
  static constexpr int kElem = kF8 ? 1 : 2;          // bytes per Q/K/V element
  static constexpr int kBM = 128;                    // rows per Q tile
  static constexpr int kBN = 128;                    // keys per KV tile
  static constexpr int kQT = kD == 256 ? 1 : 2;      // Q tiles per CTA
  static constexpr int kRows = kQT * kBM;            // query rows per CTA
  static constexpr int kChunkElems = 128 / kElem;    // elements per 128-byte row
  static constexpr int kChunks = kD / kChunkElems;   // 128-byte column chunks
  static constexpr int kChunkBytes = 128 * 128;      // 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = kTileBytes >= 65536 ? 2 : (kTileBytes >= 32768 ? 4 : 8);  // K/V ring slots
  static constexpr int kQKSteps = kD * kElem / 32;   // K-steps of QK^T (32 bytes each)
  static constexpr int kPVKeys = 32 / kElem;         // keys per K-step of PV
  static constexpr int kPVStepBytes = kPVKeys * 128; // V rows of one PV K-step
  static constexpr float kLazy = kF8 ? 4.f : 8.f;    // max growth (log2) before a rescale
  static constexpr float kPOff = kF8 ? 4.f : 0.f;    // P = 2^(x - m + kPOff)
  static constexpr int kBarOffset = (kQT + kStages) * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kBarOffset + kBarBytes + 1024;  // + barriers + align slack
  static_assert(kStages <= 8, "more ring slots than the barrier block holds");
  static constexpr int kThreads = 128 * (1 + kQT);
  // registers of warpgroup 0 (producer, MMA issuer) after setmaxnreg.dec
  // and of the softmax warpgroups after setmaxnreg.inc. With softcap or FP8
  // the producer/MMA code spills at 88, so those variants move registers to
  // it (measured against 88/208: FP8 1.4 % faster at 104/200; softcap 3 %
  // faster at 104/200 and another 1 % at 112/192, where FP8 is 2.7 % slower;
  // the plain causal forward is 0.5 % slower with either, so it keeps the
  // first split).
  static constexpr int kRegsLow = 88;
  static constexpr int kRegsHigh = 208;
  static constexpr int kRegsLowF8 = 104;
  static constexpr int kRegsHighF8 = 200;
  static constexpr int kRegsLowCap = 112;
  static constexpr int kRegsHighCap = 192;
  static constexpr int kTmemCols = 512;
  // of every 8 pairs of exponentials, this many run as a cubic on the FMA
  // pipe instead of the special-function unit (which bounds the softmax)
  static constexpr int kPolyOf8 = 2;
  // with softcap, whose tanh already loads the FMA pipe
  static constexpr int kPolyOf8Cap = 1;
  // P_t is stored and signalled in this many parts, so that PV starts on
  // the first part while the rest of the row is exponentiated
  static constexpr int kPParts = 4;
  static constexpr int kPKeys = 128 / kPParts;
  static constexpr int kPCols = kPKeys * kElem / 4;  // TMEM columns of one part of P
  static constexpr int kColS = 0;      // + 128 * t
  static constexpr int kColP = 64;     // + 128 * t
  static constexpr int kColO = 128 * kQT;  // + kD * t
};

// Barrier block in shared memory.
struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint64_t s_full[2];
  uint64_t p_ready[2][2];  // [Q tile][part 0, 1]: P of keys [32 h, 32 (h + 1)) in TMEM
  uint64_t o_final[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  // the CTA's work item, written by thread 0 during setup and read back by
  // every role after its register reallocation (so that no value crosses it)
  int item[8];
  // parts 2 and 3 of P. The placement of the barriers in this block was
  // measured to move the forward's time by about 3 %; this order is the
  // fastest of those measured.
  uint64_t p_ready_hi[2][2];
  // [t][0, 1]: the K/V tiles (indices into the CTA's n_tiles) Q tile t
  // takes part in, [first, end): a tile that the mask hides from all of its
  // rows is skipped
  int tile_range[2][2];
};

__device__ __forceinline__ uint64_t* p_ready_bar(FwdBars* b, int t, int h) {
  return h < 2 ? &b->p_ready[t][h] : &b->p_ready_hi[t][h - 2];
}

struct FwdItem {
  int seq_start, seq_len, q0, h, b, kvh, n_begin, n_tiles;
};

__device__ __forceinline__ FwdItem load_item(const FwdBars* bars) {
  const volatile int* v = bars->item;
  return FwdItem{v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]};
}

__device__ __forceinline__ bool fwd_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicExch(&g_device_status, kDevTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max (kMax) or min of 128 values, four independent chains
template <bool kMax>
__device__ __forceinline__ float reduce128(const float (&x)[128]) {
  float a[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) a[c] = x[c];
#pragma unroll
  for (int i = 4; i + 8 <= 128; i += 8) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
      a[c] = kMax ? max3(a[c], x[i + c], x[i + 4 + c]) : min3(a[c], x[i + c], x[i + 4 + c]);
  }
  // elements 124..127
#pragma unroll
  for (int c = 0; c < 4; ++c) a[c] = kMax ? fmaxf(a[c], x[124 + c]) : fminf(a[c], x[124 + c]);
  return kMax ? max3(fmaxf(a[0], a[1]), a[2], a[3]) : min3(fminf(a[0], a[1]), a[2], a[3]);
}

// kAlibi: the ALiBi bias is compiled in only where it is used, so the
// common instantiations keep their register allocation
// kBF16 is the output type (and, without kF8, the input type).
// kWithhold (only the failure-path test instantiates it): the producer never
// issues the first K tile's load, so every wait on it runs out after
// p.wait_ns and the CTA unwinds (FA_ERR_TIMEOUT in the status word) with no
// copy or MMA left in flight.
template <int kD, bool kBF16, bool kCap, bool kAlibi, bool kF8 = false, bool kWithhold = false>
__global__ void __launch_bounds__(FwdShape<kD, kF8>::kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Sh = FwdShape<kD, kF8>;
  static_assert(sizeof(FwdBars) <= Sh::kBarBytes, "barrier block exceeds its reservation");
  // The K/V tiles stream from the last (nearest the diagonal) backwards:
  // loop index it runs over physical tile n_tiles - 1 - it, and the per-Q-tile
  // ranges are kept in loop order. Under a causal mask the second Q tile sees
  // one tile more than the first, the diagonal one; taken first, that tile's
  // softmax overlaps the other Q tile's first products instead of running
  // alone before the epilogue (causal S2048 10 % and D256 8 % faster than in
  // ascending order). With ALiBi, the bias also makes the nearest keys the
  // row's largest logits, so the running max is set by the first tile and the
  // lazy rescale of O (a read-modify-write of the accumulator) is rare.
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                               // 2 tiles
  uint8_t* sKV = smem + Sh::kQT * Sh::kTileBytes;   // kStages tiles
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + Sh::kBarOffset);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  {
  // ---- work item: (sequence, head) major so the CTAs in flight share the
  // K/V of a few heads in L2; heaviest query blocks first within a head
  int b, h, qb, seq_start, seq_len;
  if (p.seq_blocks) {
    // varlen, B <= 64: sequence b owns Hq * ceil(len_b / kRows) consecutive
    // blocks, so that no block starts past its sequence's end (the grid is
    // the bound Hq * (ceil(total / kRows) + B)). Every warp finds its block's
    // sequence: lanes take sequences lane and lane + 32, and an inclusive
    // prefix sum of their block counts over the warp locates blockIdx.x.
    const unsigned full = 0xffffffffu;
    const int ln = threadIdx.x & 31;
    const int blk = static_cast<int>(blockIdx.x);
    int st[2] = {0, 0}, en[2] = {0, 0}, cnt[2] = {0, 0};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int sq = ln + 32 * u;
      if (sq < p.B) {
        st[u] = p.cu_seqlens[sq];
        en[u] = p.cu_seqlens[sq + 1];
        cnt[u] = (en[u] - st[u] + Sh::kRows - 1) / Sh::kRows * p.Hq;
      }
    }
    int inc[2] = {cnt[0], cnt[1]};
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = __shfl_up_sync(full, inc[u], off);
        if (ln >= off) inc[u] += t;
      }
    }
    inc[1] += __shfl_sync(full, inc[0], 31);
    const unsigned m0 = __ballot_sync(full, ln < p.B && inc[0] > blk);
    const unsigned m1 = __ballot_sync(full, ln + 32 < p.B && inc[1] > blk);
    if (m0 == 0u && m1 == 0u) return;  // past the last sequence's blocks (uniform, before any barrier)
    const int u = m0 != 0u ? 0 : 1;
    const int src = __ffs(static_cast<int>(m0 != 0u ? m0 : m1)) - 1;
    b = src + 32 * u;
    const int first = __shfl_sync(full, u == 0 ? inc[0] - cnt[0] : inc[1] - cnt[1], src);
    seq_start = __shfl_sync(full, u == 0 ? st[0] : st[1], src);
    seq_len = __shfl_sync(full, u == 0 ? en[0] : en[1], src) - seq_start;
    const int nq = (seq_len + Sh::kRows - 1) / Sh::kRows;
    const int rem = blk - first;
    h = rem / nq;
    qb = nq - 1 - rem % nq;
  } else {
    const int bh = static_cast<int>(blockIdx.x) / p.n_qblocks;
    qb = p.n_qblocks - 1 - static_cast<int>(blockIdx.x) % p.n_qblocks;
    h = bh % p.Hq;
    b = bh / p.Hq;
    if (p.cu_seqlens != nullptr) {
      seq_start = p.cu_seqlens[b];
      seq_len = p.cu_seqlens[b + 1] - seq_start;
    } else {
      seq_start = b * p.S;
      seq_len = p.S;
    }
  }
  const int q0 = qb * Sh::kRows;
  if (q0 >= seq_len) return;  // uniform across the CTA, before any barrier
  const int kvh = h / p.group;

  // visible key range of the whole 256-row block (self-attention: Sk = Sq)
  const int row_hi = min(q0 + Sh::kRows - 1, seq_len - 1);
  int key_hi = seq_len - 1;
  if (p.wr >= 0) key_hi = min(key_hi, row_hi + p.wr);
  int key_lo = 0;
  if (p.wl >= 0) key_lo = max(0, q0 - p.wl);
  const int n_begin = key_lo / Sh::kBN;
  const int n_end = key_hi >= key_lo ? key_hi / Sh::kBN + 1 : n_begin;
  const int n_tiles = n_end - n_begin;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < Sh::kStages; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int t = 0; t < Sh::kQT; ++t) {
      mbar_init(&bars->s_full[t], 1);
      for (int h = 0; h < Sh::kPParts; ++h) mbar_init(p_ready_bar(bars, t, h), 4);
      mbar_init(&bars->o_final[t], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    const int item[8] = {seq_start, seq_len, q0, h, b, kvh, n_begin, n_tiles};
    for (int i = 0; i < 8; ++i) bars->item[i] = item[i];
    // per Q tile: the sub-range of the CTA's K/V tiles its rows can see
    for (int t = 0; t < Sh::kQT; ++t) {
      const int r0 = q0 + t * Sh::kBM;
      int first = 0, end = 0;
      if (r0 < seq_len && n_tiles > 0) {
        const int r1 = min(r0 + Sh::kBM - 1, seq_len - 1);
        int hi = seq_len - 1;
        if (p.wr >= 0) hi = min(hi, r1 + p.wr);
        const int lo = p.wl >= 0 ? max(0, r0 - p.wl) : 0;
        if (hi >= lo) {
          first = lo / Sh::kBN - n_begin;
          end = hi / Sh::kBN + 1 - n_begin;
        }
      }
      bars->tile_range[t][0] = end > first ? n_tiles - end : first;
      bars->tile_range[t][1] = end > first ? n_tiles - first : end;
    }
    fence_mbar_init();
    // the Q tiles and the first K tile are requested here, so that their
    // latency overlaps the TMEM allocation and the block syncs below; the
    // producer starts its ring at the first V tile (the self-test withholds
    // the first K tile and so never requests it)
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    mbar_arrive_expect_tx(&bars->q_full, Sh::kQT * Sh::kTileBytes);
    for (int t = 0; t < Sh::kQT; ++t)
      for (int c = 0; c < Sh::kChunks; ++c)
        tma_load_3d(&tm_q, &bars->q_full, sQ + t * Sh::kTileBytes + c * Sh::kChunkBytes,
                    c * Sh::kChunkElems, h, seq_start + q0 + t * 128);
    if (!kWithhold && n_tiles > 0) {
      mbar_arrive_expect_tx(&bars->kv_full[0], Sh::kTileBytes);
      for (int c = 0; c < Sh::kChunks; ++c)
        tma_load_3d(&tm_k, &bars->kv_full[0], sKV + c * Sh::kChunkBytes, c * Sh::kChunkElems, kvh,
                    seq_start + (n_begin + n_tiles - 1) * Sh::kBN);
    }
  }
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, Sh::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* abort = &bars->abort;
  constexpr int kRegsLow = kCap ? Sh::kRegsLowCap : (kF8 ? Sh::kRegsLowF8 : Sh::kRegsLow);
  constexpr int kRegsHigh = kCap ? Sh::kRegsHighCap : (kF8 ? Sh::kRegsHighF8 : Sh::kRegsHigh);
  static_assert(Sh::kQT == 1 || Sh::kThreads * 168 >= 128 * kRegsLow + 256 * kRegsHigh,
                "register split exceeds the launch pool");
  static_assert(kRegsLow % 8 == 0 && kRegsHigh % 8 == 0, "setmaxnreg takes multiples of 8");
  // register reallocation sits inside each role's branch so the compiler
  // knows which limit every region runs under
  if (warp < 4) {
    // (one Q tile: 256 threads, every thread has the 255 registers it may use)
    if constexpr (Sh::kQT == 2) regs_dec<kRegsLow>();
  if (warp == 0) {
    // ======================= TMA producer =======================
    if (elect_one()) {
      const FwdItem w = load_item(bars);
      const int seq_start = w.seq_start, kvh = w.kvh;
      const int n_begin = w.n_begin, n_tiles = w.n_tiles;
      tma_prefetch_desc(&tm_v);
      int fill = 0;
      for (int j = 0; j < n_tiles && !*abort; ++j) {
        const int tok = seq_start + (n_begin + n_tiles - 1 - j) * Sh::kBN;
        for (int kv = 0; kv < 2; ++kv, ++fill) {
          const int slot = fill % Sh::kStages;
          const uint32_t ph = static_cast<uint32_t>(fill / Sh::kStages) & 1u;
          if (!fwd_wait(&bars->kv_empty[slot], ph ^ 1u, abort, p.wait_ns)) break;
          if (fill == 0) continue;  // requested at setup (withheld: neither count nor copy)
          mbar_arrive_expect_tx(&bars->kv_full[slot], Sh::kTileBytes);
          uint8_t* dst = sKV + slot * Sh::kTileBytes;
          const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
          for (int c = 0; c < Sh::kChunks; ++c)
            tma_load_3d(tm, &bars->kv_full[slot], dst + c * Sh::kChunkBytes, c * Sh::kChunkElems,
                        kvh, tok);
        }
      }
      // drain: every issued load must land before the CTA may exit
      for (int f = max(0, fill - Sh::kStages); f < fill; ++f) {
        const int slot = f % Sh::kStages;
        mbar_wait(&bars->kv_full[slot], static_cast<uint32_t>(f / Sh::kStages) & 1u, p.wait_ns);
      }
      mbar_wait(&bars->q_full, 0, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (elect_one()) {
      const int n_tiles = load_item(bars).n_tiles;
      const uint32_t tmem = *static_cast<volatile uint32_t*>(&bars->tmem_base);
      constexpr uint32_t id_qk = kF8 ? idesc_e4m3(128, 128, false, false)
                                     : idesc_f16(kBF16, 128, 128, false, false);
      constexpr uint32_t id_pv = kF8 ? idesc_e4m3(128, kD, false, true)
                                     : idesc_f16(kBF16, 128, kD, false, true);
      // descriptors are built once; a tile or K-step offset is added to the
      // start-address field (bits 0..13, in 16-byte units; every address
      // stays below 256 KB, so the addition never carries out of the field)
      const uint64_t dq_base = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk_base = sdesc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dv_base = sdesc_sw128(smem_u32(sKV), Sh::kChunkBytes, 1024);
      bool ok = fwd_wait(&bars->q_full, 0, abort, p.wait_ns);
      tc_fence_after();
      int t_first[2], t_end[2];
      for (int t = 0; t < Sh::kQT; ++t) {
        t_first[t] = static_cast<volatile int*>(bars->tile_range[t])[0];
        t_end[t] = static_cast<volatile int*>(bars->tile_range[t])[1];
      }
      auto in_range = [&](int t, int j) { return j >= t_first[t] && j < t_end[t]; };
      auto issue_qk = [&](int t, int slot) {
        const uint64_t a0 = dq_base + static_cast<uint64_t>((t * Sh::kTileBytes) >> 4);
        const uint64_t b0 = dk_base + static_cast<uint64_t>((slot * Sh::kTileBytes) >> 4);
        const uint32_t d = tmem + Sh::kColS + 128 * t;
#pragma unroll
        for (int kk = 0; kk < Sh::kQKSteps; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * Sh::kChunkBytes + (kk & 3) * 32) >> 4);
          umma_ss_k<kF8>(d, a0 + off, b0 + off, id_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V over the keys of part hf (K-steps of kPVKeys keys, each
      // 8 TMEM columns of P)
      auto issue_pv = [&](int t, int slot, int hf, bool first) {
        constexpr int kSteps = Sh::kPKeys / Sh::kPVKeys;
        const uint64_t b0 = dv_base + static_cast<uint64_t>((slot * Sh::kTileBytes) >> 4);
        const uint32_t d = tmem + Sh::kColO + kD * t;
        const uint32_t a = tmem + Sh::kColS + 128 * t + Sh::kColP;
#pragma unroll
        for (int kk = kSteps * hf; kk < kSteps * (hf + 1); ++kk)
          umma_ts_k<kF8>(d, a + kk * 8, b0 + static_cast<uint64_t>((kk * Sh::kPVStepBytes) >> 4),
                         id_pv, (first && kk == 0) ? 0u : 1u);
      };
      // every part of PV_t, each as soon as its part of P is in TMEM
      auto wait_issue_pv = [&](int t, int slot, uint32_t ph, bool first) {
        for (int hf = 0; hf < Sh::kPParts; ++hf) {
          if (!fwd_wait(p_ready_bar(bars, t, hf), ph, abort, p.wait_ns)) return false;
          tc_fence_after();
          issue_pv(t, slot, hf, first);
        }
        return true;
      };
      for (int it = 0; it < n_tiles && ok; ++it) {
        const int fk = 2 * it, fv = 2 * it + 1;
        const int sk = fk % Sh::kStages;
        if (!(ok = fwd_wait(&bars->kv_full[sk], static_cast<uint32_t>(fk / Sh::kStages) & 1u, abort, p.wait_ns)))
          break;
        tc_fence_after();
        if (it > 0) {
          const int fvp = fv - 2, svp = fvp % Sh::kStages;
          // per Q tile: PV_t of the previous K/V tile, then QK_t of this one
          // (each only inside the tile's range; a tile's output is final
          // after its last PV); the previous V slot is free after the last
          // tile's PV
          const int j = it - 1;
          for (int t = 0; t < Sh::kQT && ok; ++t) {
            if (in_range(t, j)) {
              const uint32_t ph = static_cast<uint32_t>(j - t_first[t]) & 1u;
              if (!(ok = wait_issue_pv(t, svp, ph, j == t_first[t]))) break;
              if (j == t_end[t] - 1) umma_commit(&bars->o_final[t]);
            }
            if (t == Sh::kQT - 1) umma_commit(&bars->kv_empty[svp]);
            if (in_range(t, it)) {
              issue_qk(t, sk);
              umma_commit(&bars->s_full[t]);
            }
          }
          if (!ok) break;
          umma_commit(&bars->kv_empty[sk]);
        } else {
          for (int t = 0; t < Sh::kQT; ++t) {
            if (in_range(t, 0)) {
              issue_qk(t, sk);
              umma_commit(&bars->s_full[t]);
            }
          }
          umma_commit(&bars->kv_empty[sk]);
        }
        // V_it must be resident before next round's PV
        const int sv = fv % Sh::kStages;
        if (!(ok = fwd_wait(&bars->kv_full[sv], static_cast<uint32_t>(fv / Sh::kStages) & 1u, abort, p.wait_ns)))
          break;
      }
      if (ok && n_tiles > 0) {
        const int j = n_tiles - 1;
        const int fvl = 2 * j + 1, svl = fvl % Sh::kStages;
        for (int t = 0; t < Sh::kQT && ok; ++t) {
          if (!in_range(t, j)) continue;
          const uint32_t ph = static_cast<uint32_t>(j - t_first[t]) & 1u;
          if (!(ok = wait_issue_pv(t, svl, ph, j == t_first[t]))) break;
          umma_commit(&bars->o_final[t]);
        }
        umma_commit(&bars->kv_empty[svl]);
      }
      // wait for everything this thread issued before TMEM is released
      umma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, p.wait_ns);
    }
    __syncwarp();
  }
  } else {
    if constexpr (Sh::kQT == 2) regs_inc<kRegsHigh>();
    const FwdItem w = load_item(bars);
    const uint32_t tmem = *static_cast<volatile uint32_t*>(&bars->tmem_base);
    const int seq_start = w.seq_start, seq_len = w.seq_len, q0 = w.q0, h = w.h, b = w.b;
    const int n_begin = w.n_begin;
    // ======================= softmax groups =======================
    const int t = (warp - 4) >> 2;            // Q tile of this group
    const int it_first = static_cast<volatile int*>(bars->tile_range[t])[0];
    const int it_end = static_cast<volatile int*>(bars->tile_range[t])[1];
    const int lane_base = 32 * (warp & 3);    // TMEM lanes this warp may touch
    const int row = lane_base + lane;         // row within the Q tile
    const int qrow = q0 + t * 128 + row;      // row within the sequence
    const uint32_t t_s = tmem + (static_cast<uint32_t>(lane_base) << 16) + Sh::kColS + 128 * t;
    const uint32_t t_p = t_s + Sh::kColP;
    const uint32_t t_o = tmem + (static_cast<uint32_t>(lane_base) << 16) + Sh::kColO + kD * t;
    // tile-level visibility of this 128-row tile
    const int r_lo = q0 + t * 128 + lane_base;   // this warp's first row
    const int r_hi = r_lo + 31;
    float m_run = -INFINITY;
    float l_run = 0.f;
    // ALiBi slope of this head in the exp2 domain (uniform across the CTA)
    constexpr bool alibi = kAlibi;
    const float sl2 = alibi ? p.alibi[static_cast<size_t>(b) * p.alibi_bstride + h] * 1.4426950408889634f : 0.f;
    bool ok = true;
    for (int it = it_first; it < it_end; ++it) {
      if (!(ok = fwd_wait(&bars->s_full[t], static_cast<uint32_t>(it - it_first) & 1u, abort, p.wait_ns))) break;
      tc_fence_after();
      // ---- the row of S_t: 128 raw scores ----
      float x[128];
      {
        uint32_t* u = reinterpret_cast<uint32_t*>(x);
        tmem_ld32(t_s + 0, reinterpret_cast<uint32_t(&)[32]>(u[0]));
        tmem_ld32(t_s + 32, reinterpret_cast<uint32_t(&)[32]>(u[32]));
        tmem_ld32(t_s + 64, reinterpret_cast<uint32_t(&)[32]>(u[64]));
        tmem_ld32(t_s + 96, reinterpret_cast<uint32_t(&)[32]>(u[96]));
        tmem_ld_wait();
      }
      const int k0 = (n_begin + w.n_tiles - 1 - it) * Sh::kBN;
      // does any (row, key) of this warp's 32 x 128 block need masking?
      bool need_mask = (k0 + 127 >= seq_len);
      if (p.wr >= 0) need_mask |= (k0 + 127 > r_lo + p.wr);
      if (p.wl >= 0) need_mask |= (k0 < r_hi - p.wl);
      // softcap on an unmasked tile whose |scale * s / softcap| are all below
      // kTanhCubicMax (the common case): tanh is the odd cubic s (b0 + b1 s^2)
      // with the scale and softcap folded into b0, b1, and its subtraction
      // of the row's running max fuses into the last FMA below, after the
      // tile's max, which the cubic, being monotone, takes at the raw max or
      // min. x keeps the raw scores until then.
      bool cubic = false;
      float cb[2];       // folded cubic coefficients
      float mt_cubic = 0.f;
      if constexpr (kCap && !alibi) {
        if (!need_mask) {
          float hi[4], lo[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) hi[c] = lo[c] = x[c];
#pragma unroll
          for (int i = 4; i + 8 <= 128; i += 8) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              hi[c] = max3(hi[c], x[i + c], x[i + 4 + c]);
              lo[c] = min3(lo[c], x[i + c], x[i + 4 + c]);
            }
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            hi[c] = fmaxf(hi[c], x[124 + c]);
            lo[c] = fminf(lo[c], x[124 + c]);
          }
          const float smax = max3(fmaxf(hi[0], hi[1]), hi[2], hi[3]);
          const float smin = min3(fminf(lo[0], lo[1]), lo[2], lo[3]);
          cubic = __all_sync(0xffffffffu, fmaxf(smax, -smin) * fabsf(p.cap_in) <= kTanhCubicMax);
          if (cubic) {
            fold_tanh(kTanhCubic, p.cap_in, p.cap_out_log2, cb);
            mt_cubic = fmaxf(smax * fmaf(cb[1], smax * smax, cb[0]), smin * fmaf(cb[1], smin * smin, cb[0]));
          }
        }
      }
      if (kCap && !cubic) {
        // logits in the exp2 domain: softcap * tanh(scale * s / softcap) * log2(e).
        // When every |scale * s / softcap| of the warp's rows is small, tanh
        // is an FMA-pipe polynomial with the scale and softcap folded into
        // its coefficients (two values per instruction; degree 2 below 1/4,
        // degree 4 below 1/2); otherwise the exp-based identity.
        float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 128; i += 8) {
#pragma unroll
          for (int c = 0; c < 4; ++c) am[c] = max3(am[c], fabsf(x[i + c]), fabsf(x[i + 4 + c]));
        }
        const float ya = max3(fmaxf(am[0], am[1]), am[2], am[3]) * fabsf(p.cap_in);
        if (__all_sync(0xffffffffu, ya <= kTanhPolyMaxLo)) {
          float pk[3];
          fold_tanh(kTanhLo, p.cap_in, p.cap_out_log2, pk);
#pragma unroll
          for (int i = 0; i < 128; i += 2) {
            const float2 v = tanh_fold2(make_float2(x[i], x[i + 1]), pk);
            x[i] = v.x;
            x[i + 1] = v.y;
          }
        } else if (__all_sync(0xffffffffu, ya <= kTanhPolyMax)) {
          float pk[5];
          fold_tanh(kTanhHi, p.cap_in, p.cap_out_log2, pk);
#pragma unroll
          for (int i = 0; i < 128; i += 2) {
            const float2 v = tanh_fold2(make_float2(x[i], x[i + 1]), pk);
            x[i] = v.x;
            x[i + 1] = v.y;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 128; ++i) x[i] = p.cap_out_log2 * tanh_fast(x[i] * p.cap_in);
        }
      }
      if constexpr (alibi) {
        // ALiBi: -slope * |query - key| added to the logit, in the exp2
        // domain (after softcap); x then holds exp2-domain logits. When every
        // key of the tile lies on one side of every row of the warp (always,
        // for the visible keys of a causal tile), the bias is affine in the
        // key index i, c + d * i, and costs one packed FMA per pair; a tile
        // that straddles the warp's rows takes the absolute value per key.
        const float dq = static_cast<float>(qrow - k0);
        const bool left = p.wr == 0 || k0 + 127 <= r_lo;  // keys at or before the rows
        const bool right = k0 >= r_hi;                     // keys at or after the rows
        if (__all_sync(0xffffffffu, left || right)) {
          const float c = left ? -sl2 * dq : sl2 * dq;
          const float d = left ? sl2 : -sl2;
          const float2 c2 = make_float2(c, c), d2 = make_float2(d, d);
          const float2 sc2 = make_float2(kCap ? 1.f : p.scale_log2, kCap ? 1.f : p.scale_log2);
#pragma unroll
          for (int i = 0; i < 128; i += 2) {
            const float2 bias = __ffma2_rn(make_float2(static_cast<float>(i), static_cast<float>(i + 1)), d2, c2);
            const float2 v = __ffma2_rn(make_float2(x[i], x[i + 1]), sc2, bias);
            x[i] = v.x;
            x[i + 1] = v.y;
          }
        } else if constexpr (kCap) {
#pragma unroll
          for (int i = 0; i < 128; ++i) x[i] = fmaf(-sl2, fabsf(dq - static_cast<float>(i)), x[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            x[i] = fmaf(x[i], p.scale_log2, -sl2 * fabsf(dq - static_cast<float>(i)));
        }
      }
      constexpr bool lg = kCap || alibi;  // x holds exp2-domain logits
      // masked entries become the value that the reduction ignores and whose
      // exponential is 0 (-inf; +inf for raw scores under a negative scale)
      const bool pos = lg || p.scale_log2 >= 0.f;
      if (need_mask) {
        const float hide = pos ? -INFINITY : INFINITY;
        int jmax = seq_len - 1 - k0;
        if (p.wr >= 0) jmax = min(jmax, qrow + p.wr - k0);
        const int jmin = p.wl >= 0 ? qrow - p.wl - k0 : INT32_MIN;
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] = (i > jmax || i < jmin) ? hide : x[i];
      }
      float mt;
      if (cubic) {
        mt = mt_cubic;
      } else if constexpr (lg) {
        mt = reduce128<true>(x);
      } else {
        mt = pos ? reduce128<true>(x) : reduce128<false>(x);
        mt *= p.scale_log2;  // +-inf stays -inf for a fully masked row
        if (mt != mt) mt = -INFINITY;
      }
      const float m_new = fmaxf(m_run, mt);
      const bool grow = m_new > m_run + Sh::kLazy;
      if (__any_sync(0xffffffffu, grow)) {
        const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m_run - m_new);
        if (m_new != -INFINITY) m_run = m_new;
        l_run *= alpha;
        if (it > it_first) {
          // O_t holds the previous PV results (complete: s_full commit
          // follows them); rescale it in place
#pragma unroll 1
          for (int c = 0; c < kD / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(t_o + c * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(t_o + c * 16, r);
          }
        }
      }
      const float base = (m_run == -INFINITY) ? 0.f : m_run - Sh::kPOff;
      // P = 2^(x - base): one packed FMA (or add) per pair, then the
      // exponentials, 64 at a time, all issued before any of their results is
      // used so that they pipeline through the special-function unit
      const float2 nb2 = make_float2(-base, -base);
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
      if (kCap && !alibi && cubic) {
        // raw scores: s (b0 + b1 s^2) - base, three packed operations a pair
        // (cb is set only in the variants that compile the cubic in)
        if constexpr (kCap && !alibi) {
          const float2 b0 = make_float2(cb[0], cb[0]), b1 = make_float2(cb[1], cb[1]);
#pragma unroll
          for (int i = 0; i < 128; i += 2) {
            const float2 xv = make_float2(x[i], x[i + 1]);
            const float2 q = __ffma2_rn(__fmul2_rn(xv, xv), b1, b0);
            const float2 d = __ffma2_rn(q, xv, nb2);
            x[i] = d.x;
            x[i + 1] = d.y;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 128; i += 2) {
          const float2 xv = make_float2(x[i], x[i + 1]);
          const float2 d = lg ? __fadd2_rn(xv, nb2) : __ffma2_rn(xv, sc2, nb2);
          x[i] = d.x;
          x[i + 1] = d.y;
        }
      }
      // the parts of the row in turn: their exponentials, then their 16-bit
      // P into TMEM and a signal, so that the tensor core starts on the first
      // part of PV while the rest is exponentiated
      float2 sum2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
      for (int hf = 0; hf < Sh::kPParts; ++hf) {
        float* xh = x + Sh::kPKeys * hf;
#pragma unroll
        for (int i = 0; i < Sh::kPKeys; i += 2) {
          if (((i >> 1) & 7) < (kCap ? Sh::kPolyOf8Cap : Sh::kPolyOf8)) {
            const float2 e = ex2_poly2(make_float2(xh[i], xh[i + 1]));
            xh[i] = e.x;
            xh[i + 1] = e.y;
          } else {
            xh[i] = ex2_approx(xh[i]);
            xh[i + 1] = ex2_approx(xh[i + 1]);
          }
        }
        uint32_t r[Sh::kPCols];
        if constexpr (kF8) {
#pragma unroll
          for (int i = 0; i < Sh::kPCols; ++i) {
            r[i] = pack4_e4m3(xh[4 * i], xh[4 * i + 1], xh[4 * i + 2], xh[4 * i + 3]);
            sum2[(2 * i) & 3] = __fadd2_rn(sum2[(2 * i) & 3], make_float2(xh[4 * i], xh[4 * i + 1]));
            sum2[(2 * i + 1) & 3] =
                __fadd2_rn(sum2[(2 * i + 1) & 3], make_float2(xh[4 * i + 2], xh[4 * i + 3]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < Sh::kPCols; ++i) {
            r[i] = pack2_alu<kBF16>(xh[2 * i], xh[2 * i + 1]);
            sum2[i & 3] = __fadd2_rn(sum2[i & 3], make_float2(xh[2 * i], xh[2 * i + 1]));
          }
        }
        if constexpr (Sh::kPCols == 32)
          tmem_st32(t_p + hf * 32, r);
        else if constexpr (Sh::kPCols == 16)
          tmem_st16(t_p + hf * 16, r);
        else
          tmem_st8(t_p + hf * 8, r);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready_bar(bars, t, hf));
      }
      const float2 s01 = __fadd2_rn(sum2[0], sum2[1]), s23 = __fadd2_rn(sum2[2], sum2[3]);
      const float2 s4 = __fadd2_rn(s01, s23);
      l_run += s4.x + s4.y;
    }
    // ---- epilogue: O / l and LSE ----
    const bool any = it_end > it_first;
    if (ok && any) ok = fwd_wait(&bars->o_final[t], 0, abort, p.wait_ns);
    tc_fence_after();
    const bool valid_row = qrow < seq_len;
    const float inv_l = l_run > 0.f ? (kF8 ? p.o_scale : 1.f) / l_run : 0.f;
    typedef uint4 Vec;
    uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) +
                    (static_cast<size_t>(seq_start + qrow) * p.Hq + h) * kD * 2;
#pragma unroll 1
    for (int c = 0; c < kD / 32; ++c) {
      uint32_t r[32];
      if (ok && any) {
        tmem_ld32(t_o + c * 32, r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        w[i] = pack2<kBF16>(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
      if (valid_row) {
        Vec* dst = reinterpret_cast<Vec*>(orow + c * 64);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
    if (valid_row) {
      const float lse =
          l_run > 0.f ? (m_run - Sh::kPOff + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      const size_t li = p.cu_seqlens != nullptr
                            ? static_cast<size_t>(h) * p.total + seq_start + qrow
                            : (static_cast<size_t>(b) * p.Hq + h) * p.S + qrow;
      p.lse[li] = lse;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*static_cast<volatile uint32_t*>(&bars->tmem_base), Sh::kTmemCols);
  }
}

}  // namespace fa
