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
//   bwd_pre_kernel   Drow = rowsum(dO * O) per (token, query head); zero the
//                    float32 dQ accumulator.
//   bwd_main_kernel  one CTA per (sequence, kv head, 128-key tile); K and V
//                    stay resident while the CTA walks every query head of
//                    the GQA group and every 128-row Q tile that can see the
//                    keys, accumulating dK and dV in tensor memory; each
//                    tile's dQ contribution is staged through shared memory
//                    and added to the float32 accumulator with TMA bulk
//                    reduce-add (atomic per element in L2).
//   bwd_post_kernel  dQ accumulator -> 16-bit dq.
//
// bwd_main warp roles (320 threads):
//   warp 0     TMA producer: K, V once; Q_i and dO_i into a 2-slot ring.
//   warp 1     MMA issuer (one lane), TMEM owner.
//   warps 2-9  two compute groups; group g owns query columns [64g, 64g+64):
//              one thread per key row computes P^T = exp(S^T - LSE) and
//              dS^T = P^T * (dP^T - Drow), P^T -> TMEM (16-bit), dS^T -> smem;
//              then one thread per query row moves dQ columns [64g, 64g+64)
//              from TMEM through smem to the reduce-add; at the end group 0
//              writes dV, group 1 dK.
// TMEM columns: A [0,128) S^T then P^T (queries [64g, 64g+64) packed into
// [64g, 64g+32)); B [128,256) dP^T then dQ; dV [256, 256+D); dK [256+D, 256+2D).
#pragma once

#include "ptx.cuh"

namespace fa {

struct BwdParams {
  int B, Hq, Hkv, S, total, group;
  int n_ktiles;              // ceil(S / 128)
  float scale;               // multiplies dS (so dQ, dK come out scaled)
  float scale_log2;          // scale * log2(e)
  float softcap, cap_in, cap_out_log2;
  int wl, wr;                // window (causal folded into wr)
  const void* o;
  const void* dout;
  const float* lse;
  float* drow;               // LSE layout
  float* dq_acc;             // (T, Hq, D) float32
  void* dq;                  // (T, Hq, D) 16-bit
  void* dk;                  // (T, Hkv, D)
  void* dv;
  const int* cu_seqlens;
};

// ---------------------------------------------------------------------------
// pre: Drow and zeroed dQ accumulator. One warp per (token, head) row.
// ---------------------------------------------------------------------------
template <int kD, bool kBF16>
__global__ void bwd_pre_kernel(const BwdParams p) {
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(p.total) * p.Hq;
  if (gw >= rows) return;
  const int tok = static_cast<int>(gw / p.Hq);
  const int h = static_cast<int>(gw % p.Hq);
  constexpr int kPer = kD / 32;  // elements per lane
  const uint16_t* o = static_cast<const uint16_t*>(p.o) + gw * kD + lane * kPer;
  const uint16_t* d = static_cast<const uint16_t*>(p.dout) + gw * kD + lane * kPer;
  float acc = 0.f;
  if constexpr (kPer == 4) {
    const uint2 ov = *reinterpret_cast<const uint2*>(o);
    const uint2 dv = *reinterpret_cast<const uint2*>(d);
    const float2 o0 = unpack2<kBF16>(ov.x), o1 = unpack2<kBF16>(ov.y);
    const float2 d0 = unpack2<kBF16>(dv.x), d1 = unpack2<kBF16>(dv.y);
    acc = o0.x * d0.x + o0.y * d0.y + o1.x * d1.x + o1.y * d1.y;
  } else {
    const uint32_t ov = *reinterpret_cast<const uint32_t*>(o);
    const uint32_t dv = *reinterpret_cast<const uint32_t*>(d);
    const float2 o0 = unpack2<kBF16>(ov), d0 = unpack2<kBF16>(dv);
    acc = o0.x * d0.x + o0.y * d0.y;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  float4* z = reinterpret_cast<float4*>(p.dq_acc + gw * kD);
  for (int i = lane; i < kD / 4; i += 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane == 0) {
    size_t li;
    if (p.cu_seqlens != nullptr) {
      li = static_cast<size_t>(h) * p.total + tok;
    } else {
      const int b = tok / p.S, s = tok % p.S;
      li = (static_cast<size_t>(b) * p.Hq + h) * p.S + s;
    }
    p.drow[li] = acc;
  }
}

// ---------------------------------------------------------------------------
// post: dq = dq_acc (already scaled) -> 16-bit
// ---------------------------------------------------------------------------
template <bool kBF16>
__global__ void bwd_post_kernel(const BwdParams p, long long n4) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(p.dq_acc)[i];
  uint2 w;
  w.x = pack2<kBF16>(v.x, v.y);
  w.y = pack2<kBF16>(v.z, v.w);
  reinterpret_cast<uint2*>(p.dq)[i] = w;
}

// ---------------------------------------------------------------------------
// main
// ---------------------------------------------------------------------------
template <int kD>
struct BwdShape {
  static constexpr int kChunks = kD / 64;
  static constexpr int kChunkBytes = 128 * 128;        // 128 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kDsBytes = 2 * kChunkBytes;     // 128 keys x 128 queries x 16 bit
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;         // + slot * 2 * kTileBytes (Q, dO)
  static constexpr int kOffDs = 6 * kTileBytes;
  static constexpr int kOffVec = kOffDs + kDsBytes;    // lse_log2[128], drow[128]
  static constexpr int kOffBar = kOffVec + 1024;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static constexpr int kThreads = 320;
  static constexpr int kTmemCols = 512;
  static constexpr int kColA = 0;
  static constexpr int kColB = 128;
  static constexpr int kColDV = 256;
  static constexpr int kColDK = 256 + kD;
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t qd_full[2];
  uint64_t qd_empty[2];
  uint64_t s_ready;
  uint64_t p_ready;
  uint64_t ds_ready;
  uint64_t dq_ready;
  uint64_t dq_free;
  uint64_t final_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool bwd_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        atomicExch(&g_device_status, kDevTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

template <int kD, bool kBF16, bool kCap>
__global__ void __launch_bounds__(320, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using Sh = BwdShape<kD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + Sh::kOffBar);
  float* vec_lse = reinterpret_cast<float*>(smem + Sh::kOffVec);
  float* vec_drow = vec_lse + 128;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (sequence, kv head) major, so the CTAs in flight add into
  // the dQ rows of only a few heads (which then stay in L2); within a head,
  // key tiles in increasing order, i.e. the ones with most query tiles first
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
  // query rows that can see some key of [k0, k0 + 127]
  int q_lo = 0;
  if (p.wr >= 0) q_lo = max(0, k0 - p.wr);
  int q_hi = seq_len - 1;
  if (p.wl >= 0) q_hi = min(q_hi, k0 + 127 + p.wl);
  const int i_begin = q_lo / 128;
  const int i_cnt = q_hi >= q_lo ? q_hi / 128 + 1 - i_begin : 0;
  const int n_items = i_cnt * p.group;  // (head, q tile) pairs

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->qd_full[s], 1);
      mbar_init(&bars->qd_empty[s], 1);
    }
    mbar_init(&bars->s_ready, 1);
    mbar_init(&bars->p_ready, 8);
    mbar_init(&bars->ds_ready, 8);
    mbar_init(&bars->dq_ready, 1);
    mbar_init(&bars->dq_free, 2);
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
      mbar_arrive_expect_tx(&bars->kv_full, 2 * Sh::kTileBytes);
      for (int c = 0; c < Sh::kChunks; ++c) {
        tma_load_3d(&tm_k, &bars->kv_full, smem + Sh::kOffK + c * Sh::kChunkBytes, c * 64, kvh,
                    seq_start + k0);
        tma_load_3d(&tm_v, &bars->kv_full, smem + Sh::kOffV + c * Sh::kChunkBytes, c * 64, kvh,
                    seq_start + k0);
      }
      int it = 0;
      for (; it < n_items && !*abort; ++it) {
        const int slot = it & 1;
        const uint32_t ph = static_cast<uint32_t>(it >> 1) & 1u;
        if (!bwd_wait(&bars->qd_empty[slot], ph ^ 1u, abort)) break;
        const int h = kvh * p.group + it / i_cnt;
        const int tok = seq_start + (i_begin + it % i_cnt) * 128;
        uint8_t* dst = smem + Sh::kOffQ + slot * 2 * Sh::kTileBytes;
        mbar_arrive_expect_tx(&bars->qd_full[slot], 2 * Sh::kTileBytes);
        for (int c = 0; c < Sh::kChunks; ++c) {
          tma_load_3d(&tm_q, &bars->qd_full[slot], dst + c * Sh::kChunkBytes, c * 64, h, tok);
          tma_load_3d(&tm_do, &bars->qd_full[slot], dst + Sh::kTileBytes + c * Sh::kChunkBytes,
                      c * 64, h, tok);
        }
      }
      for (int f = max(0, it - 2); f < it; ++f)
        mbar_wait(&bars->qd_full[f & 1], static_cast<uint32_t>(f >> 1) & 1u);
      mbar_wait(&bars->kv_full, 0);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (elect_one()) {
      constexpr uint32_t id_s = idesc_f16(kBF16, 128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t id_dv = idesc_f16(kBF16, 128, kD, false, true);    // P^T (tmem) x dO
      constexpr uint32_t id_dk = idesc_f16(kBF16, 128, kD, false, true);    // dS^T x Q
      constexpr uint32_t id_dq = idesc_f16(kBF16, 128, kD, true, true);     // dS x K
      const uint32_t sK = smem_u32(smem + Sh::kOffK);
      const uint32_t sV = smem_u32(smem + Sh::kOffV);
      const uint32_t sDs = smem_u32(smem + Sh::kOffDs);
      bool ok = bwd_wait(&bars->kv_full, 0, abort);
      tc_fence_after();
      auto kmajor = [](uint32_t base, int kk) {
        return sdesc_sw128(base + (kk >> 2) * Sh::kChunkBytes + (kk & 3) * 32, 16, 1024);
      };
      auto mnmajor = [](uint32_t base, int kk) {
        return sdesc_sw128(base + kk * 2048, Sh::kChunkBytes, 1024);
      };
      auto issue_s = [&](uint32_t sQ) {
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_ss(tmem + Sh::kColA, kmajor(sK, kk), kmajor(sQ, kk), id_s, kk > 0 ? 1u : 0u);
      };
      if (ok && n_items > 0) {
        if ((ok = bwd_wait(&bars->qd_full[0], 0, abort))) {
          tc_fence_after();
          issue_s(smem_u32(smem + Sh::kOffQ));
        }
      }
      for (int it = 0; it < n_items && ok; ++it) {
        const int slot = it & 1;
        const uint32_t sQ = smem_u32(smem + Sh::kOffQ + slot * 2 * Sh::kTileBytes);
        const uint32_t sDO = sQ + Sh::kTileBytes;
        // region B must be free: the dQ group has read the previous dQ
        if (it > 0) {
          if (!(ok = bwd_wait(&bars->dq_free, static_cast<uint32_t>(it - 1) & 1u, abort))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_ss(tmem + Sh::kColB, kmajor(sV, kk), kmajor(sDO, kk), id_s, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_ready);
        if (!(ok = bwd_wait(&bars->p_ready, static_cast<uint32_t>(it) & 1u, abort))) break;
        tc_fence_after();
        const uint32_t acc_first = (it == 0) ? 0u : 1u;
        // dV += P^T dO (A = P^T from TMEM region A: queries [64g, 64g+64) are
        // packed into columns [64g, 64g+32), 16 queries = 8 columns per step)
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          umma_ts(tmem + Sh::kColDV, tmem + Sh::kColA + (kk >> 2) * 64 + (kk & 3) * 8, mnmajor(sDO, kk), id_dv,
                  (kk == 0) ? acc_first : 1u);
        // dK += dS^T Q (after dS^T is in shared memory)
        if (!(ok = bwd_wait(&bars->ds_ready, static_cast<uint32_t>(it) & 1u, abort))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          umma_ss(tmem + Sh::kColDK, kmajor(sDs, kk), mnmajor(sQ, kk), id_dk,
                  (kk == 0) ? acc_first : 1u);
        // dQ = dS K  -> region B
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          umma_ss(tmem + Sh::kColB, mnmajor(sDs, kk), mnmajor(sK, kk), id_dq, kk > 0 ? 1u : 0u);
        umma_commit(&bars->dq_ready);
        umma_commit(&bars->qd_empty[slot]);
        // next S^T into region A (P^T of this item has been consumed in order)
        if (it + 1 < n_items) {
          const int ns = (it + 1) & 1;
          if (!(ok = bwd_wait(&bars->qd_full[ns], static_cast<uint32_t>((it + 1) >> 1) & 1u, abort)))
            break;
          tc_fence_after();
          issue_s(smem_u32(smem + Sh::kOffQ + ns * 2 * Sh::kTileBytes));
        }
      }
      umma_commit(&bars->final_done);
      umma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    // ======================= compute groups =======================
    // Group g (warps 2-5: g = 0; warps 6-9: g = 1) owns query columns
    // [64g, 64g+64) of S^T and dP^T (one thread per key row), and columns
    // [64g, 64g+64) of each dQ tile (one thread per query row).
    const int g = (warp - 2) >> 2;
    const int lane_base = 32 * (warp & 3);
    const int r = lane_base + lane;
    const int key = k0 + r;
    const int gt = static_cast<int>(threadIdx.x) - 64 - 128 * g;  // 0..127 in the group
    const uint32_t lane_off = static_cast<uint32_t>(lane_base) << 16;
    const uint32_t t_a = tmem + lane_off + Sh::kColA;
    const uint32_t t_b = tmem + lane_off + Sh::kColB;
    float* glse = vec_lse + 64 * g;
    float* gdrow = vec_drow + 64 * g;
    const uint32_t bar_id = 2u + static_cast<uint32_t>(g);
    // the group's query-row vectors of item `it` (threads 0..63: LSE in the
    // exp2 domain; 64..127: Drow), loaded one item ahead
    auto load_vec = [&](int it) -> float {
      float v = gt < 64 ? INFINITY : 0.f;
      if (it < n_items) {
        const int h = kvh * p.group + it / i_cnt;
        const int qi = (i_begin + it % i_cnt) * 128 + 64 * g + (gt & 63);
        if (qi < seq_len) {
          const size_t li = p.cu_seqlens != nullptr
                                ? static_cast<size_t>(h) * p.total + seq_start + qi
                                : (static_cast<size_t>(b) * p.Hq + h) * p.S + qi;
          if (gt < 64) {
            const float l = p.lse[li];
            v = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
          } else {
            v = p.drow[li];
          }
        }
      }
      return v;
    };
    float nv = load_vec(0);
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int it = 0; it < n_items; ++it) {
      const int h = kvh * p.group + it / i_cnt;
      const int i0 = (i_begin + it % i_cnt) * 128;
      named_bar_sync(bar_id, 128);  // the group is done with the previous vectors
      if (gt < 64)
        glse[gt] = nv;
      else
        gdrow[gt - 64] = nv;
      named_bar_sync(bar_id, 128);
      nv = load_vec(it + 1);
      if (!(ok = bwd_wait(&bars->s_ready, static_cast<uint32_t>(it) & 1u, abort))) break;
      tc_fence_after();
      // does any (key, query) of this warp's 32 keys x the group's 64 queries need masking?
      const int kw_lo = k0 + lane_base, kw_hi = kw_lo + 31;
      const int qg_lo = i0 + 64 * g, qg_hi = qg_lo + 63;
      bool need_mask = (kw_hi >= seq_len) || (qg_hi >= seq_len);
      if (p.wr >= 0) need_mask |= (kw_hi > qg_lo + p.wr);
      if (p.wl >= 0) need_mask |= (kw_lo < qg_hi - p.wl);
      // pass 1: P^T from S^T (32 queries per chunk) -> TMEM; keep
      // w = P * scale (* (1 - tanh^2) under softcap) for the dS pass
      float w[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * g + cc;       // chunk index within the 128 queries
        uint32_t sr[32];
        tmem_ld32(t_a + c * 32, sr);
        tmem_ld_wait();
        bool poly = false;
        if constexpr (kCap) {
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(sr[i])), fabsf(__uint_as_float(sr[i + 1]))));
          poly = __all_sync(0xffffffffu, amax * fabsf(p.cap_in) <= kTanhPolyMax);
        }
        uint32_t pk[16];
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const int jl = cc * 32 + 2 * j2;  // query within the group
          const float2 s2 = make_float2(__uint_as_float(sr[2 * j2]), __uint_as_float(sr[2 * j2 + 1]));
          const float2 l2 = *reinterpret_cast<const float2*>(glse + jl);
          float2 arg, fac;
          if constexpr (kCap) {
            float2 th;
            if (poly)
              th = tanh_poly2(__fmul2_rn(s2, make_float2(p.cap_in, p.cap_in)));
            else
              th = make_float2(tanh_fast(s2.x * p.cap_in), tanh_fast(s2.y * p.cap_in));
            arg = make_float2(p.cap_out_log2 * th.x - l2.x, p.cap_out_log2 * th.y - l2.y);
            fac = make_float2((1.f - th.x * th.x) * p.scale, (1.f - th.y * th.y) * p.scale);
          } else {
            arg = __ffma2_rn(s2, sc2, make_float2(-l2.x, -l2.y));
            fac = make_float2(p.scale, p.scale);
          }
          float2 pr = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
          if (need_mask) {
            const int q0i = qg_lo + jl;
            bool v0 = key < seq_len && q0i < seq_len;
            bool v1 = key < seq_len && q0i + 1 < seq_len;
            if (p.wr >= 0) {
              v0 = v0 && key <= q0i + p.wr;
              v1 = v1 && key <= q0i + 1 + p.wr;
            }
            if (p.wl >= 0) {
              v0 = v0 && key >= q0i - p.wl;
              v1 = v1 && key >= q0i + 1 - p.wl;
            }
            pr.x = v0 ? pr.x : 0.f;
            pr.y = v1 ? pr.y : 0.f;
          }
          pk[j2] = pack2<kBF16>(pr.x, pr.y);
          const float2 wv = __fmul2_rn(pr, fac);
          w[jl] = wv.x;
          w[jl + 1] = wv.y;
        }
        // P^T of queries [32c, 32c+32) -> TMEM region A columns [64g + 16cc, +16):
        // only columns this group has already read are overwritten
        tmem_st16(t_a + 64 * g + 16 * cc, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready);  // dV may start
      // pass 2: dS^T = w * (dP^T - Drow) -> shared memory (the dK and dQ operand)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * g + cc;
        uint32_t dr[32];
        tmem_ld32(t_b + c * 32, dr);
        tmem_ld_wait();
        uint32_t dsk[16];
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const int jl = cc * 32 + 2 * j2;
          const float2 dp2 = make_float2(__uint_as_float(dr[2 * j2]), __uint_as_float(dr[2 * j2 + 1]));
          const float2 d2 = *reinterpret_cast<const float2*>(gdrow + jl);
          const float2 ds = __fmul2_rn(__fadd2_rn(dp2, make_float2(-d2.x, -d2.y)), make_float2(w[jl], w[jl + 1]));
          dsk[j2] = pack2<kBF16>(ds.x, ds.y);
        }
        // dS^T row r, queries [32c, 32c+32): 64-query chunk g, 16-byte groups 4cc..4cc+3
        uint8_t* rowp = smem + Sh::kOffDs + g * Sh::kChunkBytes + r * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int gg = cc * 4 + q4;
          *reinterpret_cast<uint4*>(rowp + ((gg ^ (r & 7)) << 4)) =
              make_uint4(dsk[4 * q4], dsk[4 * q4 + 1], dsk[4 * q4 + 2], dsk[4 * q4 + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready);

      // ---- dQ tile: TMEM -> shared-memory staging -> TMA reduce-add ----
      // The staging slot is this group's half of the dS^T buffer: dq_ready
      // follows the dK and dQ MMAs that read dS^T, and the next dS^T is only
      // written after dq_free (both groups) has let the next dP^T MMA run.
      if (!(ok = bwd_wait(&bars->dq_ready, static_cast<uint32_t>(it) & 1u, abort))) break;
      tc_fence_after();
      uint8_t* stage = smem + Sh::kOffDs + g * Sh::kChunkBytes;
      const bool valid = i0 + r < seq_len;
#pragma unroll 1
      for (int cc = 0; cc < kD / 64; ++cc) {
        const int c = (kD / 64) * g + cc;  // 32-column dQ chunk
        uint32_t rr[32];
        tmem_ld32(t_b + c * 32, rr);
        tmem_ld_wait();
        if (cc > 0) {
          if (gt == 0) bulk_wait_read<0>();  // previous chunk has left the slot
          named_bar_sync(bar_id, 128);
        }
        uint8_t* rowp = stage + r * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 v = valid ? make_uint4(rr[4 * j], rr[4 * j + 1], rr[4 * j + 2], rr[4 * j + 3])
                                : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(rowp + ((j ^ (r & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        named_bar_sync(bar_id, 128);
        if (gt == 0) {
          tma_reduce_add_3d(&tm_dq, stage, c * 32, h, seq_start + i0);
          bulk_commit();
        }
      }
      if (gt == 0) bulk_wait_read<0>();
      tc_fence_before();
      named_bar_sync(bar_id, 128);
      if (gt == 0) mbar_arrive(&bars->dq_free);
    }
    if (gt == 0) bulk_wait<0>();  // every reduction has reached global memory

    // ---- epilogue: group 0 writes the dV rows, group 1 the dK rows ----
    if (ok) ok = bwd_wait(&bars->final_done, 0, abort);
    tc_fence_after();
    void* outp = g == 0 ? p.dv : p.dk;
    const uint32_t col = g == 0 ? Sh::kColDV : Sh::kColDK;
    uint8_t* dst = static_cast<uint8_t*>(outp) + (static_cast<size_t>(seq_start + key) * p.Hkv + kvh) * kD * 2;
    if (ok && n_items > 0) {
      // every lane loads (the TMEM load is warp-collective); only rows of
      // the sequence are stored
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_off + col + c * 32, rr);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack2<kBF16>(__uint_as_float(rr[2 * i]), __uint_as_float(rr[2 * i + 1]));
        if (key < seq_len) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
    } else if (ok && key < seq_len) {
      uint4* d4 = reinterpret_cast<uint4*>(dst);
      for (int i = 0; i < kD / 8; ++i) d4[i] = make_uint4(0u, 0u, 0u, 0u);
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
