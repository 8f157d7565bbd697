// Attention forward on the sm_100a tensor cores (tcgen05), one CTA per
// (sequence, head, 128-query tile).
//
// Heads are independent (Megatron-LM show notes: self-attention is split by
// head, so each partition runs its own heads without communication), so a CTA
// reads the Q, K, V columns of one head of one partition's fused projection.
//
//   warp 4      TMA producer: the Q tile once, then K and V tiles of 64 keys
//               into rings of 2 stages (4 at head dims up to 64; 128-byte
//               swizzle, 64-column sub-tiles).
//   warp 5      MMA issuer (whole warp, one lane issues): S_j = Q K_j^T
//               into TMEM buffer j % 2 (M=128 queries, N=64 keys), then
//               O += P_{j-1} V_{j-1} (M=128, N=head_dim) with P read from
//               tensor memory once the softmax warps have written it.
//   warps 0..3  softmax: thread r owns query row r.  It reads its S row from
//               TMEM, keeps a running max m and sum l, and writes
//               P = exp(S - m) as bf16 back into the first 32 columns of the
//               same S buffer (P_j aliases S_j, so P is double-buffered with
//               S and never touches shared memory).  Only when the running
//               max grew by more than 2^8 does it rescale its O row, and only
//               then does it wait for the previous O += P V.  At the end it
//               normalises O by l and stores O and lse (base 2, of the
//               scaled scores).
// Two CTAs share an SM (97 KB of shared memory and 256 TMEM columns each), so
// one CTA's MMAs and loads overlap the other's softmax.
//
// S and O never leave the SM; HBM traffic is Q, K, V in and O, lse out.
#include <string.h>

#include <atomic>

#include "gemm.cuh"
#include "kernels.cuh"
#include "tp_common.cuh"

namespace tp {

namespace {

// 2^x with the special-function unit's approximate exponential (PTX
// ex2.approx.ftz.f32: relative error about 2^-22; results below the normal
// range flush to zero; 2^-inf = 0).  For softmax weights that are rounded to
// bf16 or summed in fp32 this is exact enough and saves the range handling
// of exp2f.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


constexpr int kTileQ = 128;
constexpr int kTileK = 64;
constexpr uint32_t kSubTileBytes = 128 * 128;   // 128 rows x 64 bf16, one swizzle column block
constexpr uint32_t kKSubBytes = kTileK * 128;   // 64 rows x 64 bf16
constexpr int kSoftmaxThreads = 128;
constexpr int kAttnThreads = kSoftmaxThreads + 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct AttnMaps {
  CUtensorMap q[8];    // box 64 x 128 rows
  CUtensorMap kv[8];   // box 64 x 64 rows
};

struct AttnTcParams {
  int batch, seq, heads, hp, d, causal;
  float scale_log2;
  const int32_t* valid_len;
  __nv_bfloat16* o[8];
  float* lse;
  DropSite drop;   // attention-probability dropout (thresh 0: none)
  int head0, heads_total;   // dropout rows: (b * heads_total + head0 + head) * seq + q
};

// smem layout (offsets from a 1024-aligned base)
constexpr uint32_t kOffQ = 0;                                 // 2 sub-tiles of 128 rows
// K and V rings: 4 x kKSubBytes each, 2 stages of 2 sub-tiles (head dims
// above 64) or 4 stages of one (head dims up to 64)
constexpr uint32_t kOffK = kOffQ + 2 * kSubTileBytes;
constexpr uint32_t kOffV = kOffK + 4 * kKSubBytes;
constexpr uint32_t kOffBar = kOffV + 4 * kKSubBytes;
constexpr size_t kAttnSmem = 1024 + kOffBar + 256;

// TMEM columns: S buffers at 0 and 64 (P_j, bf16, in the first 32 columns of
// S_j once the softmax has read it), O at 128.
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;

__device__ __forceinline__ int valid_keys_tc(const int32_t* valid_len, int b, int seq) {
  if (!valid_len) return seq;
  const int v = valid_len[b];
  return v < 0 ? 0 : (v > seq ? seq : v);
}

template <int D, bool DROP>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_fwd_tc_kernel(const __grid_constant__ AttnMaps maps, const __grid_constant__ AttnTcParams p) {
  constexpr int NSUB = (D + 63) / 64;
  constexpr int NSTG = NSUB == 1 ? 4 : 2;   // K / V ring depth
  constexpr uint32_t IDESC_S = make_idesc_bf16(kTileQ, kTileK, false, false);
  constexpr uint32_t IDESC_PV = make_idesc_bf16(kTileQ, D, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [NSTG]
  uint64_t* k_empty = bars + 5;   // [NSTG]
  uint64_t* v_full = bars + 9;    // [NSTG]
  uint64_t* v_empty = bars + 13;  // [NSTG]
  uint64_t* s_full = bars + 17;   // [2] S_j computed
  uint64_t* s_free = bars + 19;   // [2] O += P_j V_j done: buffer j % 2 may take S_{j+2}
  uint64_t* p_full = bars + 21;   // [2] P_j written (and O rescaled if it had to be)
  uint64_t* o_ready = bars + 23;  // O += P_j V_j done (one phase per j)
  // O complete (one phase, after the last PV).  The final wait cannot use
  // o_ready: two products may still be outstanding then, and a parity wait
  // cannot tell "two phases behind" from "done".
  uint64_t* o_done = bars + 24;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 25);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (batch * heads, query tiles): blocks go out x-fastest, so every
  // head's last (longest causal) query tile is dispatched before any shorter one
  const int qt = gridDim.y - 1 - blockIdx.y;
  const int b = blockIdx.x / p.heads, head = blockIdx.x % p.heads;
  const int part = head / p.hp, lh = head % p.hp;
  const int q0 = qt * kTileQ;
  const int n_valid = valid_keys_tc(p.valid_len, b, p.seq);
  int kv_end = n_valid;
  if (p.causal) kv_end = min(kv_end, q0 + kTileQ);
  const int n_tiles = (kv_end + kTileK - 1) / kTileK;
  const int row_tok = b * p.seq;                    // token index of position 0
  const int col_q = lh * D;
  const int col_k = p.hp * D + lh * D;
  const int col_v = 2 * p.hp * D + lh * D;
  const CUtensorMap* qmap = &maps.q[part];
  const CUtensorMap* kvmap = &maps.kv[part];

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < NSTG; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), 1);
      mbar_init(smem_u32(&p_full[i]), kSoftmaxThreads);
    }
    mbar_init(smem_u32(o_ready), 1);
    mbar_init(smem_u32(o_done), 1);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0 && n_tiles > 0) {
      // ------------------------------------------------------------ TMA producer
      tma_prefetch_desc(qmap);
      tma_prefetch_desc(kvmap);
      mbar_arrive_expect_tx(smem_u32(q_full), NSUB * kSubTileBytes);
      for (int s = 0; s < NSUB; ++s)
        tma_load_2d(smem_u32(sm + kOffQ + s * kSubTileBytes), qmap, col_q + 64 * s, row_tok + q0,
                    smem_u32(q_full));
      // K_j and V_j into stage j % NSTG of their rings; V lags K by one
      // tile (O += P V of tile j runs after S of tile j + 1 is issued).
      for (int j = 0; j < n_tiles; ++j) {
        const int ks = j % NSTG;
        const uint32_t ph = (j / NSTG) & 1;
        if (!mbar_wait(smem_u32(&k_empty[ks]), ph ^ 1, DEV_ERR_TIMEOUT_EMPTY, 20)) break;
        mbar_arrive_expect_tx(smem_u32(&k_full[ks]), NSUB * kKSubBytes);
        for (int s = 0; s < NSUB; ++s)
          tma_load_2d(smem_u32(sm + kOffK + (ks * NSUB + s) * kKSubBytes), kvmap, col_k + 64 * s,
                      row_tok + j * kTileK, smem_u32(&k_full[ks]));
        if (!mbar_wait(smem_u32(&v_empty[ks]), ph ^ 1, DEV_ERR_TIMEOUT_EMPTY, 21)) break;
        mbar_arrive_expect_tx(smem_u32(&v_full[ks]), NSUB * kKSubBytes);
        for (int s = 0; s < NSUB; ++s)
          tma_load_2d(smem_u32(sm + kOffV + (ks * NSUB + s) * kKSubBytes), kvmap, col_v + 64 * s,
                      row_tok + j * kTileK, smem_u32(&v_full[ks]));
      }
    }
  } else if (warp == 5) {
    const uint32_t iss = elect_one();
    if (n_tiles > 0) {
      // ------------------------------------------------------------ MMA issuer (whole warp, one lane issues)
      // Issue order S_0, S_1, PV_0, S_2, PV_1, ...: S_j is issued after
      // PV_{j-2}, and a completed S_j therefore implies a completed PV_{j-2}
      // (the softmax warps rely on this for their o_ready parity).
      const uint32_t aq = smem_u32(sm + kOffQ);
      bool ok = mbar_wait_warp(smem_u32(q_full), 0, DEV_ERR_TIMEOUT_FULL, 22);
      auto issue_pv = [&](int j) -> bool {
        const int st = j & 1, ks = j % NSTG;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait_warp(smem_u32(&p_full[st]), ph, DEV_ERR_TIMEOUT_FULL, 23)) return false;
        if (!mbar_wait_warp(smem_u32(&v_full[ks]), (j / NSTG) & 1, DEV_ERR_TIMEOUT_FULL, 24)) return false;
        tc_fence_after();
        const uint32_t av = smem_u32(sm + kOffV + ks * NSUB * kKSubBytes);
        const uint32_t ap = tmem + st * kTileK;   // P_j: 128 rows x 64 keys, bf16 pairs
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk) {
          const uint64_t bd = sw128_desc(av + kk * 2048, kKSubBytes, 1024);
          tc_mma_bf16_ts_if(iss, tmem + kColO, ap + kk * 8, bd, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit_if(iss, smem_u32(o_ready));
        tc_commit_if(iss, smem_u32(&v_empty[ks]));
        tc_commit_if(iss, smem_u32(&s_free[st]));
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j & 1, ks = j % NSTG;
        if (!mbar_wait_warp(smem_u32(&k_full[ks]), (j / NSTG) & 1, DEV_ERR_TIMEOUT_FULL, 25) ||
            !mbar_wait_warp(smem_u32(&s_free[st]), ((j >> 1) & 1) ^ 1, DEV_ERR_TIMEOUT_ACC, 26)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ak = smem_u32(sm + kOffK + ks * NSUB * kKSubBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t col = (kk & 3) * 32;
          tc_mma_bf16_if(iss, tmem + st * kTileK, sw128_desc(aq + (kk >> 2) * kSubTileBytes + col, 16, 1024),
                      sw128_desc(ak + (kk >> 2) * kKSubBytes + col, 16, 1024), IDESC_S,
                      kk > 0 ? 1u : 0u);
        }
        tc_commit_if(iss, smem_u32(&s_full[st]));
        tc_commit_if(iss, smem_u32(&k_empty[ks]));
        if (j >= 1 && !issue_pv(j - 1)) ok = false;
      }
      if (ok && issue_pv(n_tiles - 1)) tc_commit_if(iss, smem_u32(o_done));
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int r = threadIdx.x;                 // query row within the tile
    const int q = q0 + r;
    const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
    const float scale = p.scale_log2;
    float m = -INFINITY, l = 0.f;              // m in scaled log2 units
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j & 1;
      if (!mbar_wait_warp(smem_u32(&s_full[st]), (j >> 1) & 1, DEV_ERR_TIMEOUT_ACC, 27)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // The whole S row: both TMEM loads in flight, one wait.
      uint32_t sv[kTileK / 32][32];
      static_assert(kTileK == 64, "the S row is two 32-column loads");
      tmem_ld32x2_wait(tmem + t_lane + st * kTileK, sv[0], tmem + t_lane + st * kTileK + 32, sv[1]);
      float x[kTileK];
#pragma unroll
      for (int c = 0; c < kTileK; ++c) x[c] = __uint_as_float(sv[c >> 5][c & 31]);
      const int k0 = j * kTileK;
      const bool need_mask = (k0 + kTileK > n_valid) || (p.causal && k0 + kTileK - 1 > q0);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < kTileK; ++c) {
          const int key = k0 + c;
          if (key >= n_valid || (p.causal && key > q)) x[c] = -INFINITY;
        }
      }
      // Row max of the raw scores (the scale is positive), 8 independent chains.
      float mxp[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxp[u] = x[u];
#pragma unroll
      for (int c = 8; c < kTileK; ++c) mxp[c & 7] = fmaxf(mxp[c & 7], x[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                             fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]))) * scale;
      // Lazy rescaling: keep the reference max unless the row max grew by more
      // than 2^8 (P stays <= 256, exact in bf16's exponent range).
      float alpha = 1.f;
      if (mx > m + kRescaleThreshold || m == -INFINITY) {
        alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - mx);
        m = mx;
        l *= alpha;
      }
      const float msafe = (m == -INFINITY) ? 0.f : m;
      float lp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // 8 independent sums
      uint32_t pw[kTileK / 2];
      if constexpr (!DROP) {
#pragma unroll
        for (int c = 0; c < kTileK / 2; ++c) {
          const float p0 = ex2_approx(fmaf(x[2 * c], scale, -msafe));
          const float p1 = ex2_approx(fmaf(x[2 * c + 1], scale, -msafe));
          lp[(2 * c) & 7] += p0;
          lp[(2 * c + 1) & 7] += p1;
          pw[c] = pack_bf16(p0, p1);
        }
      } else {
        // dropout: O takes P * keep / (1 - p); the normaliser l keeps all of P
        const uint32_t drow = static_cast<uint32_t>((b * p.heads_total + p.head0 + head) * p.seq + q);
        const uint32_t keep[2] = {drop_keep32(p.drop, drow, static_cast<uint32_t>(k0)),
                                  drop_keep32(p.drop, drow, static_cast<uint32_t>(k0 + 32))};
        const float ds = p.drop.scale;
#pragma unroll
        for (int c = 0; c < kTileK / 2; ++c) {
          const float p0 = ex2_approx(fmaf(x[2 * c], scale, -msafe));
          const float p1 = ex2_approx(fmaf(x[2 * c + 1], scale, -msafe));
          lp[(2 * c) & 7] += p0;
          lp[(2 * c + 1) & 7] += p1;
          const uint32_t kb = keep[c >> 4] >> ((2 * c) & 31);
          pw[c] = pack_bf16((kb & 1u) ? p0 * ds : 0.f, (kb & 2u) ? p1 * ds : 0.f);
        }
      }
      l += ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
      // P_j over the first 32 columns of S_j (already read into registers).
      tmem_st_32x32b_x32(tmem + t_lane + st * kTileK, pw);
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O holds sum_{i<j} P_i V_i: wait for the last of those products
        // (S_j complete implies PV_{j-2} complete, so the parity of
        // PV_{j-1} is unambiguous), then scale the row.
        if (!mbar_wait_warp(smem_u32(o_ready), (j - 1) & 1, DEV_ERR_TIMEOUT_ACC, 28)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32_wait(tmem + t_lane + kColO + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st_32x32b_x32(tmem + t_lane + kColO + c * 32, v);
        }
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full[st]));
    }
    // Output: O / l and lse = m + log2(l), in base-2 units of the scaled
    // scores (the backward forms P = 2^(s * scale * log2(e) - lse) from it).
    if (ok && n_tiles > 0 && mbar_wait_warp(smem_u32(o_done), 0, DEV_ERR_TIMEOUT_ACC, 29)) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o[part] + (long long)(row_tok + q) * (p.hp * D) + lh * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32_wait(tmem + t_lane + kColO + c * 32, v);
        if (q < p.seq) {
          uint4* o4 = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int g = 0; g < 4; ++g)
            o4[g] = make_uint4(
                pack_bf16(__uint_as_float(v[8 * g]) * inv_l, __uint_as_float(v[8 * g + 1]) * inv_l),
                pack_bf16(__uint_as_float(v[8 * g + 2]) * inv_l, __uint_as_float(v[8 * g + 3]) * inv_l),
                pack_bf16(__uint_as_float(v[8 * g + 4]) * inv_l, __uint_as_float(v[8 * g + 5]) * inv_l),
                pack_bf16(__uint_as_float(v[8 * g + 6]) * inv_l, __uint_as_float(v[8 * g + 7]) * inv_l));
        }
      }
      if (q < p.seq)
        p.lse[((long long)b * p.heads + head) * p.seq + q] =
            l > 0.f ? m + log2f(l) : -INFINITY;
    } else if (n_tiles == 0 && q < p.seq) {
      // no visible key: O = 0, lse = -inf
      __nv_bfloat16* orow = p.o[part] + (long long)(row_tok + q) * (p.hp * D) + lh * D;
      for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
      p.lse[((long long)b * p.heads + head) * p.seq + q] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool DROP>
int fwd_tc_inst(const AttnArgs& a, cudaStream_t s) {
  static std::atomic<unsigned long long> configured{0};   // one bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<D, DROP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kAttnSmem));
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const int hp = a.heads / a.t;
  const long long tokens = (long long)a.batch * a.seq;
  AttnMaps maps;
  memset(&maps, 0, sizeof(maps));
  AttnTcParams prm;
  memset(&prm, 0, sizeof(prm));
  for (int i = 0; i < a.t; ++i) {
    if (!make_map(&maps.q[i], a.qkv[i], 3LL * hp * D, tokens, 3LL * hp * D, kTileQ) ||
        !make_map(&maps.kv[i], a.qkv[i], 3LL * hp * D, tokens, 3LL * hp * D, kTileK))
      return cudaErrorInvalidValue;
    prm.o[i] = static_cast<__nv_bfloat16*>(a.o[i]);
  }
  prm.batch = a.batch;
  prm.seq = a.seq;
  prm.heads = a.heads;
  prm.hp = hp;
  prm.d = D;
  prm.causal = a.causal;
  prm.scale_log2 = kLog2e / sqrtf(static_cast<float>(D));
  prm.valid_len = a.valid_len;
  prm.lse = a.lse;
  prm.drop = a.drop;
  prm.head0 = a.head0;
  prm.heads_total = a.heads_total > 0 ? a.heads_total : a.heads;
  dim3 grid(a.batch * a.heads, (a.seq + kTileQ - 1) / kTileQ);
  attn_fwd_tc_kernel<D, DROP><<<grid, kAttnThreads, kAttnSmem, s>>>(maps, prm);
  return cudaGetLastError();
}

}  // namespace

int launch_attention_fwd_tc(const AttnArgs& a, cudaStream_t s) {
  const bool drop = a.drop.thresh != 0;
  switch (a.head_dim) {
    case 64: return drop ? fwd_tc_inst<64, true>(a, s) : fwd_tc_inst<64, false>(a, s);
    case 96: return drop ? fwd_tc_inst<96, true>(a, s) : fwd_tc_inst<96, false>(a, s);
    case 128: return drop ? fwd_tc_inst<128, true>(a, s) : fwd_tc_inst<128, false>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tp

// =========================================================================
// Attention backward on tcgen05.
//
//   dK/dV kernel: one CTA per (sequence, head, 128-key tile); for every
//     64-query tile it forms S^T = K Q^T and dP^T = V dO^T in TMEM (two
//     buffers), the elementwise warps turn them into P^T = exp(S^T / sqrt(d)
//     - lse) and dS^T = P^T (dP^T - delta) in swizzled shared memory, and the
//     MMA warp accumulates dV += P^T dO and dK += dS^T Q in TMEM.  The Q / dO
//     tiles serve as K-major operands of the first two products and as
//     MN-major operands of the last two.
//   Head dims up to 96 (fused dQ): the same CTA also forms dQ^T = K^T dS^T
//     per query tile, and dedicated warps add it into an fp32 dQ accumulator
//     with global reductions; a small kernel first computes delta =
//     rowsum(dO * O) and clears the accumulator's rows in the same pass,
//     another converts the accumulator to bf16 afterwards.  S, dP and the
//     exponentials are formed once.
//   Head dim 128 (no TMEM columns left for dQ^T): a separate dQ kernel, one
//     CTA per (sequence, head, 128-query tile); for every 64-key tile: S =
//     Q K^T, dP = dO V^T, dS = P (dP - delta), dQ += dS K.  It runs first:
//     its threads own query rows, so each computes
//     delta = rowsum(dO * O) for its row and stores it for the dK/dV kernel.
// No row reduction is needed (P comes from the saved lse), so two warps share
// each TMEM lane quarter and split the 64 columns: 8 elementwise warps per CTA.
// =========================================================================

namespace tp {
namespace {



constexpr uint32_t kBwdSub64 = 64 * 128;     // 64 rows x 64 bf16
constexpr uint32_t kBwdSub128 = 128 * 128;   // 128 rows x 64 bf16
constexpr int kBwdEwThreads = 256;           // 8 elementwise warps
constexpr int kBwdThreads = kBwdEwThreads + 64;
constexpr int kBwdProducerWarp = 8;
constexpr int kBwdMmaWarp = 9;

struct AttnBwdMaps {
  CUtensorMap qkv128[8];   // qkv buffer, box 64 x 128 rows
  CUtensorMap qkv64[8];    // qkv buffer, box 64 x 64 rows
  CUtensorMap do128[8];    // dO buffer, box 64 x 128 rows
  CUtensorMap do64[8];     // dO buffer, box 64 x 64 rows
  CUtensorMap dqacc[8];    // fp32 dQ accumulator, box head_dim x 64 rows (fused path)
};

struct AttnBwdParams {
  int batch, seq, heads, hp, causal;
  float scale_log2, scale;
  const int32_t* valid_len;
  const float* lse;
  float* delta;                 // written by the dQ kernel, read by the dK/dV kernel
  float* colsum;                // [t][batch * ceil(seq/32)][3*hp*D] column partials of dQKV
  const __nv_bfloat16* o[8];    // forward output O_i [tokens][hp*D]
  const __nv_bfloat16* d_o[8];  // its gradient dO_i
  __nv_bfloat16* dqkv[8];
  float* dq_acc[8];             // fused path: fp32 dQ_i accumulator [tokens][hp*D], unscaled
  DropSite drop;                // attention-probability dropout (thresh 0: none)
  int head0, heads_total;       // dropout rows: (b * heads_total + head0 + head) * seq + q
  int n_sms;                    // SMs of the device (fused path: L2 prefetch of the next CTA)
};

// Pull one box of a tensor map into L2: no shared-memory destination and no
// completion to wait for; the coordinates follow the tiled loads' rules.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// Store 32 floats (columns [32*half, 32*half+32) of a 64-column row) as bf16
// into a 128-byte-swizzled K-major tile.
__device__ __forceinline__ void store_half_row_sw128(uint8_t* tile, int row, int half,
                                                     const float (&v)[32]) {
  uint8_t* base = tile + row * 128;
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = half * 4 + cc;
    const uint4 w = make_uint4(pack_bf16(v[8 * cc], v[8 * cc + 1]), pack_bf16(v[8 * cc + 2], v[8 * cc + 3]),
                               pack_bf16(v[8 * cc + 4], v[8 * cc + 5]),
                               pack_bf16(v[8 * cc + 6], v[8 * cc + 7]));
    *reinterpret_cast<uint4*>(base + ((c ^ (row & 7)) << 4)) = w;
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&v)[32], float scale) {
  uint4* o4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int g = 0; g < 4; ++g)
    o4[g] = make_uint4(pack_bf16(__uint_as_float(v[8 * g]) * scale, __uint_as_float(v[8 * g + 1]) * scale),
                       pack_bf16(__uint_as_float(v[8 * g + 2]) * scale, __uint_as_float(v[8 * g + 3]) * scale),
                       pack_bf16(__uint_as_float(v[8 * g + 4]) * scale, __uint_as_float(v[8 * g + 5]) * scale),
                       pack_bf16(__uint_as_float(v[8 * g + 6]) * scale, __uint_as_float(v[8 * g + 7]) * scale));
}

// ---------------------------------------------------------------- dK / dV (head dim 128)

constexpr uint32_t kA_OffK = 0;                          // 2 x 128-row sub-tiles
constexpr uint32_t kA_OffV = kA_OffK + 2 * kBwdSub128;
constexpr int kBwdStages = 3;                            // Q/dO (dK/dV kernels) and K/V (dQ kernel) ring
constexpr uint32_t kA_OffQ = kA_OffV + 2 * kBwdSub128;   // stages x 2 x 64-row sub-tiles
constexpr uint32_t kA_OffDO = kA_OffQ + 2 * kBwdStages * kBwdSub64;
constexpr uint32_t kA_OffPT = kA_OffDO + 2 * kBwdStages * kBwdSub64;  // 128 keys x 64 queries
constexpr uint32_t kA_OffDS = kA_OffPT + kBwdSub128;
constexpr uint32_t kA_OffLD = kA_OffDS + kBwdSub128;     // [stages][lse 64 | delta 64] fp32
constexpr uint32_t kA_OffBar = kA_OffLD + kBwdStages * 128 * 4;
constexpr size_t kA_Smem = 1024 + kA_OffBar + 256;

// P^T = exp2(S^T scale - lse) and dS^T = P^T (dP^T - delta) for one thread's
// key row and 32 query columns (half `half` of a 64-query tile starting at
// q0), packed as bf16 pairs.  Masked (padding key, query past the sequence
// end, causal) entries are 0;
// with dropout, P^T takes the kept entries scaled by 1 / (1 - p) and the
// gradient w.r.t. the undropped P is the dropped dP^T likewise scaled.
template <bool DROP>
__device__ __forceinline__ void bwd_scores_t(const AttnBwdParams& p, const uint32_t (&sv)[32],
                                             const uint32_t (&dv)[32], const float* lds, int b,
                                             int head, int qh, int key, bool key_ok, bool need_mask,
                                             uint32_t (&pt)[16], uint32_t (&ds)[16]) {
  if constexpr (!DROP) {
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      float p0 = ex2_approx(fmaf(__uint_as_float(sv[c]), p.scale_log2, -lds[c]));
      float p1 = ex2_approx(fmaf(__uint_as_float(sv[c + 1]), p.scale_log2, -lds[c + 1]));
      if (need_mask) {
        if (!key_ok || qh + c >= p.seq || (p.causal && qh + c < key)) p0 = 0.f;
        if (!key_ok || qh + c + 1 >= p.seq || (p.causal && qh + c + 1 < key)) p1 = 0.f;
      }
      pt[c >> 1] = pack_bf16(p0, p1);
      ds[c >> 1] = pack_bf16(p0 * (__uint_as_float(dv[c]) - lds[64 + c]),
                             p1 * (__uint_as_float(dv[c + 1]) - lds[64 + c + 1]));
    }
  } else {
    const uint32_t drow0 = static_cast<uint32_t>((b * p.heads_total + p.head0 + head) * p.seq + qh);
    const uint32_t kg = static_cast<uint32_t>(key) >> 2, kw = static_cast<uint32_t>(key) & 3u;
    const float dsc = p.drop.scale;
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      float pv[2], dd[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float v = ex2_approx(fmaf(__uint_as_float(sv[c + u]), p.scale_log2, -lds[c + u]));
        if (need_mask && (!key_ok || qh + c + u >= p.seq || (p.causal && qh + c + u < key))) v = 0.f;
        const bool kept = (drop_keep4(p.drop, drow0 + c + u, kg) >> kw) & 1u;
        pv[u] = kept ? v * dsc : 0.f;
        dd[u] = v * ((kept ? __uint_as_float(dv[c + u]) * dsc : 0.f) - lds[64 + c + u]);
      }
      pt[c >> 1] = pack_bf16(pv[0], pv[1]);
      ds[c >> 1] = pack_bf16(dd[0], dd[1]);
    }
  }
}

// The lse and delta of the 64 queries of a step starting at q0 into lds[0..63]
// and lds[64..127], copied asynchronously (each lane its two queries); the
// lane's arrival on `bar` happens when its copies have landed, so the
// producer never waits for global memory.  Queries past the sequence end
// read as 0 (the elementwise warps mask them).
__device__ __forceinline__ void load_step_stats(const AttnBwdParams& p, long long stat0, int q0,
                                                float* lds, int lane, uint32_t bar) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = lane + 32 * h, q = q0 + c;
    const bool ok = q < p.seq;
    const float* src_l = ok ? p.lse + stat0 + q : p.lse;
    const float* src_d = ok ? p.delta + stat0 + q : p.delta;
    cp_async4(smem_u32(lds + c), src_l, ok ? 4u : 0u);
    cp_async4(smem_u32(lds + 64 + c), src_d, ok ? 4u : 0u);
  }
  cp_async_mbar_arrive(bar);
}

// 16 bf16 pairs (columns [32*half, 32*half+32) of a 64-column row) into a
// 128-byte-swizzled K-major tile.
__device__ __forceinline__ void store_half_row_packed(uint8_t* tile, int row, int half,
                                                      const uint32_t (&w)[16]) {
  uint8_t* base = tile + row * 128;
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = half * 4 + cc;
    *reinterpret_cast<uint4*>(base + ((c ^ (row & 7)) << 4)) =
        make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
  }
}

// dV (warps 0-3) or dK (warps 4-7, times the softmax scale) of this thread's
// key row from TMEM into dQKV, and the warp's column partials of the 32-row
// block (the K / V part of db_qkv).
template <int D>
__device__ __forceinline__ void bwd_store_dkdv(const AttnBwdParams& p, uint32_t tmem, uint32_t t_lane,
                                               uint32_t col_dv, uint32_t col_dk, int quarter,
                                               int half, int lane, int b, int part, int lh,
                                               int row_tok, int k0, int key) {
  const long long ldq = 3LL * p.hp * D;
  const int nrb = (p.seq + 31) / 32;
  __nv_bfloat16* rowp = p.dqkv[part] + (long long)(row_tok + key) * ldq + lh * D + (2 - half) * p.hp * D;
  const uint32_t col = half ? col_dk : col_dv;
  const float scale = half ? p.scale : 1.f;
  const int rb = (k0 + quarter * 32) / 32;   // this warp's 32-row block
  float* cs = p.colsum + ((long long)part * p.batch * nrb + b * nrb + rb) * ldq +
              (2 - half) * p.hp * D + lh * D;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t v[32];
    tmem_ld32_wait(tmem + t_lane + col + c * 32, v);
    if (key < p.seq) store_bf16x32(rowp + c * 32, v, scale);
    float f[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) f[e] = key < p.seq ? __uint_as_float(v[e]) * scale : 0.f;
    warp_colsum32(f);
    if (rb < nrb) cs[c * 32 + lane] = f[0];
  }
}

// A key tile with no valid key (key padding): dK = dV = 0, and so are their
// column partials.
template <int D>
__device__ __forceinline__ void bwd_zero_key_tile(const AttnBwdParams& p, int b, int part, int lh,
                                                  int row_tok, int k0) {
  const long long ldq = 3LL * p.hp * D;
  const int nrb = (p.seq + 31) / 32;
  __nv_bfloat16* dqkv = p.dqkv[part];
  for (int c = threadIdx.x; c < 128 * D / 8; c += blockDim.x) {
    const int r = c / (D / 8), cc = (c % (D / 8)) * 8;
    if (k0 + r < p.seq) {
      __nv_bfloat16* rowp = dqkv + (long long)(row_tok + k0 + r) * ldq + lh * D + cc;
      *reinterpret_cast<uint4*>(rowp + p.hp * D) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(rowp + 2 * p.hp * D) = make_uint4(0, 0, 0, 0);
    }
  }
  for (int c = threadIdx.x; c < 4 * 2 * D; c += blockDim.x) {
    const int blk = c / (2 * D), col = c % (2 * D);
    const int rb = k0 / 32 + blk;
    if (rb < nrb)
      p.colsum[((long long)part * p.batch * nrb + b * nrb + rb) * ldq + (col < D ? p.hp * D : 2 * p.hp * D) +
               lh * D + (col % D)] = 0.f;
  }
}

// TMEM: two S^T/dP^T buffers at 0 and 128 (S^T in the first 64 columns), dV
// at 256, dK at 384.
template <int D, bool DROP>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ AttnBwdMaps maps,
                            const __grid_constant__ AttnBwdParams p) {
  constexpr int NSUB = (D + 63) / 64;
  constexpr int BQ = 64;
  constexpr uint32_t IDESC_S = make_idesc_bf16(128, BQ, false, false);
  constexpr uint32_t IDESC_G = make_idesc_bf16(128, D, false, true);
  constexpr uint32_t kColDV = 256, kColDK = 384;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kA_OffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;                 // [kBwdStages]
  uint64_t* q_empty = bars + 1 + kBwdStages;   // [kBwdStages]
  uint64_t* s_full = bars + 1 + 2 * kBwdStages;    // [2]
  uint64_t* s_free = bars + 3 + 2 * kBwdStages;    // [2]
  uint64_t* p_full = bars + 5 + 2 * kBwdStages;
  uint64_t* pd_free = bars + 6 + 2 * kBwdStages;
  uint64_t* acc_done = bars + 7 + 2 * kBwdStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8 + 2 * kBwdStages);
  float* ld_s = reinterpret_cast<float*>(sm + kA_OffLD);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (batch * heads, key tiles): every head's first key tile (the most
  // query tiles under a causal mask) is dispatched before any later one
  const int b = blockIdx.x / p.heads, head = blockIdx.x % p.heads;
  const int part = head / p.hp, lh = head % p.hp;
  const int k0 = blockIdx.y * 128;
  const int n_valid = valid_keys_tc(p.valid_len, b, p.seq);
  const int row_tok = b * p.seq;

  if (k0 >= n_valid) {
    bwd_zero_key_tile<D>(p, b, part, lh, row_tok, k0);
    return;
  }
  const int q_begin = p.causal ? k0 : 0;
  const int n_qt = (p.seq - q_begin + BQ - 1) / BQ;
  const long long stat0 = ((long long)b * p.heads + head) * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(kv_full), 1);
    for (int i = 0; i < kBwdStages; ++i) {
      mbar_init(smem_u32(&q_full[i]), 1 + 32);
      mbar_init(smem_u32(&q_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), kBwdEwThreads);
    }
    mbar_init(smem_u32(p_full), kBwdEwThreads);
    mbar_init(smem_u32(pd_free), 1);
    mbar_init(smem_u32(acc_done), 1);
    fence_barrier_init();
  }
  if (warp == kBwdMmaWarp) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kBwdProducerWarp) {
    // -------------------------------------------------------------- producer (whole warp)
    const CUtensorMap* m128 = &maps.qkv128[part];
    const CUtensorMap* m64 = &maps.qkv64[part];
    const CUtensorMap* dmap = &maps.do64[part];
    if (lane == 0) {
      mbar_arrive_expect_tx(smem_u32(kv_full), 2 * NSUB * kBwdSub128);
      for (int s = 0; s < NSUB; ++s) {
        tma_load_2d(smem_u32(sm + kA_OffK + s * kBwdSub128), m128, p.hp * D + lh * D + 64 * s,
                    row_tok + k0, smem_u32(kv_full));
        tma_load_2d(smem_u32(sm + kA_OffV + s * kBwdSub128), m128, 2 * p.hp * D + lh * D + 64 * s,
                    row_tok + k0, smem_u32(kv_full));
      }
    }
    for (int i = 0; i < n_qt; ++i) {
      const int st = i % kBwdStages;
      const int q0 = q_begin + i * BQ;
      if (!mbar_wait_warp(smem_u32(&q_empty[st]), ((i / kBwdStages) & 1) ^ 1, DEV_ERR_TIMEOUT_EMPTY, 40))
        break;
      if (lane == 0) {
        mbar_arrive_expect_tx(smem_u32(&q_full[st]), 2 * NSUB * kBwdSub64);
        for (int s = 0; s < NSUB; ++s) {
          tma_load_2d(smem_u32(sm + kA_OffQ + (st * 2 + s) * kBwdSub64), m64, lh * D + 64 * s,
                      row_tok + q0, smem_u32(&q_full[st]));
          tma_load_2d(smem_u32(sm + kA_OffDO + (st * 2 + s) * kBwdSub64), dmap, lh * D + 64 * s,
                      row_tok + q0, smem_u32(&q_full[st]));
        }
      }
      load_step_stats(p, stat0, q0, ld_s + st * 128, lane, smem_u32(&q_full[st]));
    }
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      const uint32_t ak = smem_u32(sm + kA_OffK), av = smem_u32(sm + kA_OffV);
      const uint32_t apt = smem_u32(sm + kA_OffPT), ads = smem_u32(sm + kA_OffDS);
      bool ok = mbar_wait(smem_u32(kv_full), 0, DEV_ERR_TIMEOUT_FULL, 41);
      auto grads = [&](int t) -> bool {
        if (!mbar_wait(smem_u32(p_full), t & 1, DEV_ERR_TIMEOUT_FULL, 42)) return false;
        tc_fence_after();
        const int st = t % kBwdStages;
        const uint32_t aq = smem_u32(sm + kA_OffQ + st * 2 * kBwdSub64);
        const uint32_t ado = smem_u32(sm + kA_OffDO + st * 2 * kBwdSub64);
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
          tc_mma_bf16(tmem + kColDV, sw128_desc(apt + kk * 32, 16, 1024),
                      sw128_desc(ado + kk * 2048, kBwdSub64, 1024), IDESC_G, acc);
          tc_mma_bf16(tmem + kColDK, sw128_desc(ads + kk * 32, 16, 1024),
                      sw128_desc(aq + kk * 2048, kBwdSub64, 1024), IDESC_G, acc);
        }
        tc_commit(smem_u32(pd_free));
        tc_commit(smem_u32(&q_empty[st]));
        return true;
      };
      for (int i = 0; ok && i < n_qt; ++i) {
        const int st = i % kBwdStages;
        const int sb = i & 1;   // TMEM buffer
        if (!mbar_wait(smem_u32(&q_full[st]), (i / kBwdStages) & 1, DEV_ERR_TIMEOUT_FULL, 43) ||
            !mbar_wait(smem_u32(&s_free[sb]), ((i >> 1) & 1) ^ 1, DEV_ERR_TIMEOUT_ACC, 44)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aq = smem_u32(sm + kA_OffQ + st * 2 * kBwdSub64);
        const uint32_t ado = smem_u32(sm + kA_OffDO + st * 2 * kBwdSub64);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t c128 = (kk >> 2) * kBwdSub128 + (kk & 3) * 32;
          const uint32_t c64 = (kk >> 2) * kBwdSub64 + (kk & 3) * 32;
          tc_mma_bf16(tmem + sb * 128, sw128_desc(ak + c128, 16, 1024), sw128_desc(aq + c64, 16, 1024),
                      IDESC_S, kk > 0 ? 1u : 0u);
          tc_mma_bf16(tmem + sb * 128 + 64, sw128_desc(av + c128, 16, 1024),
                      sw128_desc(ado + c64, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&s_full[sb]));
        if (i >= 1 && !grads(i - 1)) ok = false;
      }
      if (ok && grads(n_qt - 1)) tc_commit(smem_u32(acc_done));
    }
  } else {
    // -------------------------------------------------------------- P^T, dS^T (row = key)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int key = k0 + r;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    const bool key_ok = key < n_valid;
    bool ok = true;
    for (int i = 0; i < n_qt; ++i) {
      const int st = i % kBwdStages;
      const int sb = i & 1;
      const int q0 = q_begin + i * BQ;
      if (!mbar_wait_warp(smem_u32(&s_full[sb]), (i >> 1) & 1, DEV_ERR_TIMEOUT_ACC, 45) ||
          !mbar_wait_warp(smem_u32(&q_full[st]), (i / kBwdStages) & 1, DEV_ERR_TIMEOUT_FULL, 46)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[32], dv[32];
      tmem_ld32x2_wait(tmem + t_lane + sb * 128 + 32 * half, sv, tmem + t_lane + sb * 128 + 64 + 32 * half,
                       dv);
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[sb]));
      const int qh = q0 + 32 * half;                    // first query of this half
      const bool need_mask = !key_ok || qh + 32 > p.seq || (p.causal && qh < k0 + 128);
      uint32_t pt[16], ds[16];
      bwd_scores_t<DROP>(p, sv, dv, ld_s + st * 128 + 32 * half, b, head, qh, key, key_ok, need_mask,
                         pt, ds);
      // P^T / dS^T of step i-1 have been read by its gradient MMAs
      if (i >= 1 && !mbar_wait_warp(smem_u32(pd_free), (i - 1) & 1, DEV_ERR_TIMEOUT_ACC, 47)) {
        ok = false;
        break;
      }
      store_half_row_packed(sm + kA_OffPT, r, half, pt);
      store_half_row_packed(sm + kA_OffDS, r, half, ds);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
    }
    // tcgen05.ld is warp-collective: every lane loads, only valid rows store.
    // Warps 0-3 write dV, warps 4-7 write dK.
    if (ok && mbar_wait_warp(smem_u32(acc_done), 0, DEV_ERR_TIMEOUT_ACC, 48)) {
      tc_fence_after();
      bwd_store_dkdv<D>(p, tmem, t_lane, kColDV, kColDK, quarter, half, lane, b, part, lh, row_tok, k0,
                        key);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- fused dK / dV / dQ (head dim <= 96)
//
// One CTA per (sequence, head, 128-key tile), walking the 64-query tiles:
//   warp 13      MMA issuer (the whole warp runs the loop, one lane issues):
//                per step i, S^T_i = K Q_i^T and dP^T_i = V dO_i^T into TMEM
//                buffer i % 2; then, once P^T/dS^T of step i-1 are in shared
//                memory, dV += P^T dO, dK += dS^T Q and dQ^T_{i-1} = K^T dS^T.
//   warps 0..7   elementwise: P^T and dS^T of a step into shared memory (two
//                warps per TMEM lane quarter, 32 query columns each).
//   warps 8..11  dQ: read dQ^T of a step out of TMEM (lane = head-dim row),
//                stage it as a [64 queries][head_dim] fp32 tile and add the
//                tile into the fp32 accumulator with one TMA reduce-add.
//   warp 12      TMA producer: K, V once; Q, dO and the rows' lse / delta per
//                step, in a kFbStages-deep ring.
// Double buffering of S^T/dP^T in TMEM lets the MMAs of one step run under
// the elementwise work of the next, and the dQ warps take the accumulator
// traffic off the elementwise warps' path.  (Element-wise global reductions
// for dQ, 226 MB of fp32 adds per 8.3B-scale layer, were measured 40 % slower
// than the staged tile reduce-adds.)
//
// TMEM: S^T/dP^T buffers at 0 and 128, dV at 256, dK at 256 + D, dQ^T at
// 256 + 2D (64 columns; 512 in all for D = 96).
constexpr int kFbDqWarp0 = 8;   // warps 0 .. kFbDqWarp0-1 are the elementwise warps
constexpr int kFbProducerWarp = 12;
constexpr int kFbMmaWarp = 13;
constexpr int kFbThreads = 14 * 32;
constexpr int kFbDqThreads = 128;

// Q / dO ring depth and P^T / dS^T buffers: with head_dim 96, a 3-deep ring
// and two P^T / dS^T buffers do not fit beside the dQ staging tile.
constexpr int kFbStages = 3;
constexpr int kFbPdBufs = 1;

template <int NSUB>
struct FbSmem {
  static constexpr uint32_t K = 0;                                   // NSUB x 128-row sub-tiles
  static constexpr uint32_t V = K + NSUB * kBwdSub128;
  static constexpr uint32_t Q = V + NSUB * kBwdSub128;              // [stage][NSUB] 64-row sub-tiles
  static constexpr uint32_t DO = Q + kFbStages * NSUB * kBwdSub64;
  static constexpr uint32_t PT = DO + kFbStages * NSUB * kBwdSub64;   // [buf] 128 keys x 64 queries
  static constexpr uint32_t DS = PT + kFbPdBufs * kBwdSub128;         // [buf]
  static constexpr uint32_t STG = DS + kFbPdBufs * kBwdSub128;        // [64 queries][<= 96] fp32
  static constexpr uint32_t LD = STG + 64 * 96 * 4;                   // [stage][lse 64 | delta 64]
  static constexpr uint32_t BAR = LD + kFbStages * 128 * 4;
  static constexpr size_t BYTES = 1024 + BAR + 256;
};
static_assert(FbSmem<2>::BYTES <= 232448, "fused attention backward exceeds 227 KB of shared memory");

template <int D, bool DROP>
__global__ void __launch_bounds__(kFbThreads, 1)
    attn_bwd_fused_tc_kernel(const __grid_constant__ AttnBwdMaps maps,
                             const __grid_constant__ AttnBwdParams p) {
  static_assert(D <= 96, "fused dQ needs 2 x head_dim + 320 TMEM columns");
  constexpr int NSUB = (D + 63) / 64;
  using L = FbSmem<NSUB>;
  constexpr int BQ = 64;
  constexpr int NS = kFbStages, NP = kFbPdBufs;
  constexpr uint32_t IDESC_S = make_idesc_bf16(128, BQ, false, false);
  constexpr uint32_t IDESC_G = make_idesc_bf16(128, D, false, true);
  constexpr uint32_t IDESC_Q = make_idesc_bf16(128, BQ, true, true);   // dQ^T = K^T dS^T
  constexpr uint32_t kColDV = 256, kColDK = 256 + D, kColDQ = 256 + 2 * D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;              // [NS] Q, dO, lse / delta of a step loaded
  uint64_t* q_empty = q_full + NS;          // [NS] the step's MMAs are done with them
  uint64_t* s_full = q_empty + NS;          // [2] S^T / dP^T of a step in TMEM buffer i % 2
  uint64_t* s_free = s_full + 2;            // [2] the elementwise warps have read buffer i % 2
  uint64_t* p_full = s_free + 2;            // [NP] P^T / dS^T of a step in smem buffer i % NP
  uint64_t* pd_free = p_full + NP;          // [NP] the gradient MMAs have read buffer i % NP
  uint64_t* dq_full = pd_free + NP;         // dQ^T of a step complete in TMEM
  uint64_t* dq_free = dq_full + 1;          // the dQ warps have read it
  uint64_t* stg_free = dq_free + 1;         // the previous reduce-add has read the staging tile
  uint64_t* stg_full = stg_free + 1;        // the staging tile is written
  uint64_t* acc_done = stg_full + 1;        // dV, dK complete (the last step's dQ^T may still run)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);
  float* ld_s = reinterpret_cast<float*>(sm + L::LD);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / p.heads, head = blockIdx.x % p.heads;
  const int part = head / p.hp, lh = head % p.hp;
  const int k0 = blockIdx.y * 128;
  const int n_valid = valid_keys_tc(p.valid_len, b, p.seq);
  const int row_tok = b * p.seq;

  if (k0 >= n_valid) {
    bwd_zero_key_tile<D>(p, b, part, lh, row_tok, k0);
    return;
  }
  const int q_begin = p.causal ? k0 : 0;
  const int n_qt = (p.seq - q_begin + BQ - 1) / BQ;
  const long long stat0 = ((long long)b * p.heads + head) * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(kv_full), 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(&q_full[i]), 1 + 32);
      mbar_init(smem_u32(&q_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), kBwdEwThreads);
    }
    for (int i = 0; i < NP; ++i) {
      mbar_init(smem_u32(&p_full[i]), kBwdEwThreads);
      mbar_init(smem_u32(&pd_free[i]), 1);
    }
    mbar_init(smem_u32(dq_full), 1);
    mbar_init(smem_u32(dq_free), kFbDqThreads);
    mbar_init(smem_u32(stg_free), 1);
    mbar_init(smem_u32(stg_full), kFbDqThreads);
    mbar_init(smem_u32(acc_done), 1);
    fence_barrier_init();
    // K and V of the tile are loaded once; start them before the TMEM
    // allocation and the block barrier so their latency overlaps the setup
    const CUtensorMap* m128 = &maps.qkv128[part];
    mbar_arrive_expect_tx(smem_u32(kv_full), 2 * NSUB * kBwdSub128);
    for (int s = 0; s < NSUB; ++s) {
      tma_load_2d(smem_u32(sm + L::K + s * kBwdSub128), m128, p.hp * D + lh * D + 64 * s, row_tok + k0,
                  smem_u32(kv_full));
      tma_load_2d(smem_u32(sm + L::V + s * kBwdSub128), m128, 2 * p.hp * D + lh * D + 64 * s,
                  row_tok + k0, smem_u32(kv_full));
    }
  }
  if (warp == kFbMmaWarp) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kFbProducerWarp) {
    // -------------------------------------------------------------- producer (whole warp)
    const CUtensorMap* m64 = &maps.qkv64[part];
    const CUtensorMap* dmap = &maps.do64[part];
    for (int i = 0; i < n_qt; ++i) {
      const int st = i % NS;
      const int q0 = q_begin + i * BQ;
      if (!mbar_wait_warp(smem_u32(&q_empty[st]), ((i / NS) & 1) ^ 1, DEV_ERR_TIMEOUT_EMPTY, 60)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(smem_u32(&q_full[st]), 2 * NSUB * kBwdSub64);
        for (int s = 0; s < NSUB; ++s) {
          tma_load_2d(smem_u32(sm + L::Q + (st * NSUB + s) * kBwdSub64), m64, lh * D + 64 * s,
                      row_tok + q0, smem_u32(&q_full[st]));
          tma_load_2d(smem_u32(sm + L::DO + (st * NSUB + s) * kBwdSub64), dmap, lh * D + 64 * s,
                      row_tok + q0, smem_u32(&q_full[st]));
        }
      }
      load_step_stats(p, stat0, q0, ld_s + st * 128, lane, smem_u32(&q_full[st]));
    }
    // One CTA per SM: the CTA that takes this SM next is, in launch order,
    // about one SM count further on.  Its K and V tiles are read by no other
    // CTA (so they are not in L2 yet); pull them into L2 now, while this
    // CTA still has its last steps to run.
    if (lane == 0 && p.n_sms > 0) {
      const int nxt = blockIdx.y * gridDim.x + blockIdx.x + p.n_sms;
      const int nx = nxt % gridDim.x, ny = nxt / gridDim.x;
      if (ny < static_cast<int>(gridDim.y)) {
        const int nb = nx / p.heads, nh = nx % p.heads;
        const int npart = nh / p.hp, nlh = nh % p.hp;
        const int nk0 = ny * 128;
        if (nk0 < valid_keys_tc(p.valid_len, nb, p.seq)) {
          const CUtensorMap* nm = &maps.qkv128[npart];
          for (int s = 0; s < NSUB; ++s) {
            tma_prefetch_l2_2d(nm, p.hp * D + nlh * D + 64 * s, nb * p.seq + nk0);
            tma_prefetch_l2_2d(nm, 2 * p.hp * D + nlh * D + 64 * s, nb * p.seq + nk0);
          }
        }
      }
    }
  } else if (warp == kFbMmaWarp) {
    {
      // -------------------------------------------------------------- MMA issuer (whole warp)
      const uint32_t iss = elect_one();
      const uint32_t ak = smem_u32(sm + L::K), av = smem_u32(sm + L::V);
      bool ok = mbar_wait_warp(smem_u32(kv_full), 0, DEV_ERR_TIMEOUT_FULL, 61);
      // dV, dK and dQ^T of step t, from P^T / dS^T buffer t % NP
      auto grads = [&](int t) -> bool {
        const int pb = t % NP, st = t % NS;
        if (!mbar_wait_warp(smem_u32(&p_full[pb]), (t / NP) & 1, DEV_ERR_TIMEOUT_FULL, 62)) return false;
        tc_fence_after();
        const uint32_t aq = smem_u32(sm + L::Q + st * NSUB * kBwdSub64);
        const uint32_t ado = smem_u32(sm + L::DO + st * NSUB * kBwdSub64);
        const uint32_t apt = smem_u32(sm + L::PT + pb * kBwdSub128);
        const uint32_t ads = smem_u32(sm + L::DS + pb * kBwdSub128);
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
          tc_mma_bf16_if(iss, tmem + kColDV, sw128_desc(apt + kk * 32, 16, 1024),
                      sw128_desc(ado + kk * 2048, kBwdSub64, 1024), IDESC_G, acc);
          tc_mma_bf16_if(iss, tmem + kColDK, sw128_desc(ads + kk * 32, 16, 1024),
                      sw128_desc(aq + kk * 2048, kBwdSub64, 1024), IDESC_G, acc);
        }
        // after the last step's dV / dK products the epilogue may read them,
        // while that step's dQ^T is still being formed
        if (t == n_qt - 1) tc_commit_if(iss, smem_u32(acc_done));
        // dQ^T of step t-1 has been read out of TMEM by the dQ warps
        if (!mbar_wait_warp(smem_u32(dq_free), (t & 1) ^ 1, DEV_ERR_TIMEOUT_ACC, 63)) return false;
        tc_fence_after();
        // A = K^T (the K tile read MN-major, 64-wide head-dim chunks 16 KB
        // apart), B = dS^T (MN-major, one 64-query chunk); 16 keys per step
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          tc_mma_bf16_if(iss, tmem + kColDQ, sw128_desc(ak + kk * 2048, kBwdSub128, 1024),
                      sw128_desc(ads + kk * 2048, kBwdSub64, 1024), IDESC_Q, kk > 0 ? 1u : 0u);
        tc_commit_if(iss, smem_u32(dq_full));
        tc_commit_if(iss, smem_u32(&pd_free[pb]));
        tc_commit_if(iss, smem_u32(&q_empty[st]));
        return true;
      };
      for (int i = 0; ok && i < n_qt; ++i) {
        const int st = i % NS;
        const int sb = i & 1;
        if (!mbar_wait_warp(smem_u32(&q_full[st]), (i / NS) & 1, DEV_ERR_TIMEOUT_FULL, 64) ||
            !mbar_wait_warp(smem_u32(&s_free[sb]), ((i >> 1) & 1) ^ 1, DEV_ERR_TIMEOUT_ACC, 65)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aq = smem_u32(sm + L::Q + st * NSUB * kBwdSub64);
        const uint32_t ado = smem_u32(sm + L::DO + st * NSUB * kBwdSub64);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t c128 = (kk >> 2) * kBwdSub128 + (kk & 3) * 32;
          const uint32_t c64 = (kk >> 2) * kBwdSub64 + (kk & 3) * 32;
          tc_mma_bf16_if(iss, tmem + sb * 128, sw128_desc(ak + c128, 16, 1024), sw128_desc(aq + c64, 16, 1024),
                      IDESC_S, kk > 0 ? 1u : 0u);
          tc_mma_bf16_if(iss, tmem + sb * 128 + 64, sw128_desc(av + c128, 16, 1024),
                      sw128_desc(ado + c64, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit_if(iss, smem_u32(&s_full[sb]));
        if (i >= 1 && !grads(i - 1)) ok = false;
      }
      if (ok) grads(n_qt - 1);
    }
  } else if (warp >= kFbDqWarp0) {
    // -------------------------------------------------------------- dQ accumulation
    // Lanes of a TMEM quarter are head-dim rows of dQ^T; each step's tile is
    // staged as [64 queries][D] fp32 and added with one TMA reduce-add, issued
    // by the first dQ thread once all 128 have written.
    const int quarter = warp & 3;
    const int d = quarter * 32 + lane;
    const bool rows_ok = quarter * 32 < D;   // warp-uniform: rows >= D of dQ^T are padding
    const bool leader = threadIdx.x == kFbDqWarp0 * 32;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    float* stg = reinterpret_cast<float*>(sm + L::STG);
    for (int i = 0; i < n_qt; ++i) {
      if (!mbar_wait_warp(smem_u32(dq_full), i & 1, DEV_ERR_TIMEOUT_ACC, 66)) break;
      tc_fence_after();
      uint32_t qa[32], qb[32];
      if (rows_ok) tmem_ld32x2_wait(tmem + t_lane + kColDQ, qa, tmem + t_lane + kColDQ + 32, qb);
      tc_fence_before();
      mbar_arrive(smem_u32(dq_free));
      if (leader) {
        bulk_wait_group_read0();   // the previous reduce-add has read the staging tile
        mbar_arrive(smem_u32(stg_free));
      }
      if (!mbar_wait_warp(smem_u32(stg_free), i & 1, DEV_ERR_TIMEOUT_ACC, 67)) break;
      if (rows_ok) {
#pragma unroll
        for (int c = 0; c < 32; ++c) stg[c * D + d] = __uint_as_float(qa[c]);
#pragma unroll
        for (int c = 0; c < 32; ++c) stg[(32 + c) * D + d] = __uint_as_float(qb[c]);
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(stg_full));
      if (leader && mbar_wait(smem_u32(stg_full), i & 1, DEV_ERR_TIMEOUT_ACC, 68)) {
        tma_reduce_add_2d(&maps.dqacc[part], smem_u32(stg), lh * D, row_tok + q_begin + i * BQ);
        bulk_commit_group();
      }
    }
    if (leader) bulk_wait_group0();   // reduce-adds complete before the CTA exits
  } else {
    // -------------------------------------------------------------- P^T, dS^T (row = key)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int key = k0 + r;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    const bool key_ok = key < n_valid;
    bool ok = true;
    for (int i = 0; i < n_qt; ++i) {
      const int st = i % NS;
      const int sb = i & 1, pb = i % NP;
      const int q0 = q_begin + i * BQ;
      if (!mbar_wait_warp(smem_u32(&s_full[sb]), (i >> 1) & 1, DEV_ERR_TIMEOUT_ACC, 69) ||
          !mbar_wait_warp(smem_u32(&q_full[st]), (i / NS) & 1, DEV_ERR_TIMEOUT_FULL, 70)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[32], dv[32];
      tmem_ld32x2_wait(tmem + t_lane + sb * 128 + 32 * half, sv, tmem + t_lane + sb * 128 + 64 + 32 * half,
                       dv);
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[sb]));
      const int qh = q0 + 32 * half;
      const bool need_mask = !key_ok || qh + 32 > p.seq || (p.causal && qh < k0 + 128);
      uint32_t pt[16], ds[16];
      bwd_scores_t<DROP>(p, sv, dv, ld_s + st * 128 + 32 * half, b, head, qh, key, key_ok, need_mask,
                         pt, ds);
      // buffer pb was last read by the gradient MMAs of step i - NP
      if (i >= NP &&
          !mbar_wait_warp(smem_u32(&pd_free[pb]), ((i / NP) - 1) & 1, DEV_ERR_TIMEOUT_ACC, 71)) {
        ok = false;
        break;
      }
      store_half_row_packed(sm + L::PT + pb * kBwdSub128, r, half, pt);
      store_half_row_packed(sm + L::DS + pb * kBwdSub128, r, half, ds);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full[pb]));
    }
    if (ok && mbar_wait_warp(smem_u32(acc_done), 0, DEV_ERR_TIMEOUT_ACC, 72)) {
      tc_fence_after();
      bwd_store_dkdv<D>(p, tmem, t_lane, kColDV, kColDK, quarter, half, lane, b, part, lh, row_tok, k0,
                        key);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kFbMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dQ

constexpr uint32_t kB_OffQ = 0;                           // 2 x 128-row sub-tiles
constexpr uint32_t kB_OffDO = kB_OffQ + 2 * kBwdSub128;
constexpr uint32_t kB_OffK = kB_OffDO + 2 * kBwdSub128;   // stages x 2 x 64-row sub-tiles
constexpr uint32_t kB_OffV = kB_OffK + 2 * kBwdStages * kBwdSub64;
constexpr uint32_t kB_OffDS = kB_OffV + 2 * kBwdStages * kBwdSub64;    // 128 queries x 64 keys
constexpr uint32_t kB_OffDelta = kB_OffDS + kBwdSub128;                  // [2 halves][128] fp32
constexpr uint32_t kB_OffBar = kB_OffDelta + 2 * 128 * 4;
constexpr size_t kB_Smem = 1024 + kB_OffBar + 256;

template <int D, bool DROP>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ AttnBwdMaps maps,
                          const __grid_constant__ AttnBwdParams p) {
  constexpr int NSUB = (D + 63) / 64;
  constexpr int BK = 64;
  constexpr uint32_t IDESC_S = make_idesc_bf16(128, BK, false, false);
  constexpr uint32_t IDESC_G = make_idesc_bf16(128, D, false, true);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kB_OffBar);
  uint64_t* qd_full = bars + 0;
  uint64_t* kv_full = bars + 1;                  // [kBwdStages]
  uint64_t* kv_empty = bars + 1 + kBwdStages;    // [kBwdStages]
  uint64_t* s_full = bars + 1 + 2 * kBwdStages;  // [2]
  uint64_t* s_free = bars + 3 + 2 * kBwdStages;  // [2]
  uint64_t* p_full = bars + 5 + 2 * kBwdStages;
  uint64_t* ds_free = bars + 6 + 2 * kBwdStages;
  uint64_t* acc_done = bars + 7 + 2 * kBwdStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8 + 2 * kBwdStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (batch * heads, query tiles): blocks go out x-fastest, so every
  // head's last (longest causal) query tile is dispatched before any shorter one
  const int qt = gridDim.y - 1 - blockIdx.y;
  const int b = blockIdx.x / p.heads, head = blockIdx.x % p.heads;
  const int part = head / p.hp, lh = head % p.hp;
  const int q0 = qt * 128;
  const int n_valid = valid_keys_tc(p.valid_len, b, p.seq);
  int kv_end = n_valid;
  if (p.causal) kv_end = min(kv_end, q0 + 128);
  const int n_kt = (kv_end + BK - 1) / BK;
  const int row_tok = b * p.seq;
  const long long ldq = 3LL * p.hp * D;
  const long long stat0 = ((long long)b * p.heads + head) * p.seq;
  __nv_bfloat16* dqkv = p.dqkv[part];

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(qd_full), 1);
    for (int i = 0; i < kBwdStages; ++i) {
      mbar_init(smem_u32(&kv_full[i]), 1);
      mbar_init(smem_u32(&kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), kBwdEwThreads);
    }
    mbar_init(smem_u32(p_full), kBwdEwThreads);
    mbar_init(smem_u32(ds_free), 1);
    mbar_init(smem_u32(acc_done), 1);
    fence_barrier_init();
  }
  if (warp == kBwdMmaWarp) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // S/dP buffers at 0 / 128 (+64), dQ at 256

  if (warp == kBwdProducerWarp) {
    if (lane == 0 && n_kt > 0) {
      // -------------------------------------------------------------- TMA producer
      const CUtensorMap* m128 = &maps.qkv128[part];
      const CUtensorMap* m64 = &maps.qkv64[part];
      const CUtensorMap* dmap = &maps.do128[part];
      mbar_arrive_expect_tx(smem_u32(qd_full), 2 * NSUB * kBwdSub128);
      for (int s = 0; s < NSUB; ++s) {
        tma_load_2d(smem_u32(sm + kB_OffQ + s * kBwdSub128), m128, lh * D + 64 * s, row_tok + q0,
                    smem_u32(qd_full));
        tma_load_2d(smem_u32(sm + kB_OffDO + s * kBwdSub128), dmap, lh * D + 64 * s, row_tok + q0,
                    smem_u32(qd_full));
      }
      for (int j = 0; j < n_kt; ++j) {
        const int st = j % kBwdStages;
        if (!mbar_wait(smem_u32(&kv_empty[st]), ((j / kBwdStages) & 1) ^ 1, DEV_ERR_TIMEOUT_EMPTY, 50))
          break;
        mbar_arrive_expect_tx(smem_u32(&kv_full[st]), 2 * NSUB * kBwdSub64);
        for (int s = 0; s < NSUB; ++s) {
          tma_load_2d(smem_u32(sm + kB_OffK + (st * 2 + s) * kBwdSub64), m64,
                      p.hp * D + lh * D + 64 * s, row_tok + j * BK, smem_u32(&kv_full[st]));
          tma_load_2d(smem_u32(sm + kB_OffV + (st * 2 + s) * kBwdSub64), m64,
                      2 * p.hp * D + lh * D + 64 * s, row_tok + j * BK, smem_u32(&kv_full[st]));
        }
      }
    }
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0 && n_kt > 0) {
      // -------------------------------------------------------------- MMA issuer
      const uint32_t aq = smem_u32(sm + kB_OffQ), ado = smem_u32(sm + kB_OffDO);
      const uint32_t ads = smem_u32(sm + kB_OffDS);
      bool ok = mbar_wait(smem_u32(qd_full), 0, DEV_ERR_TIMEOUT_FULL, 51);
      auto grad = [&](int t) -> bool {
        if (!mbar_wait(smem_u32(p_full), t & 1, DEV_ERR_TIMEOUT_FULL, 52)) return false;
        tc_fence_after();
        const int st = t % kBwdStages;
        const uint32_t ak = smem_u32(sm + kB_OffK + st * 2 * kBwdSub64);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma_bf16(tmem + 256, sw128_desc(ads + kk * 32, 16, 1024),
                      sw128_desc(ak + kk * 2048, kBwdSub64, 1024), IDESC_G,
                      (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(smem_u32(ds_free));
        tc_commit(smem_u32(&kv_empty[st]));
        return true;
      };
      for (int j = 0; ok && j < n_kt; ++j) {
        const int st = j % kBwdStages;
        const int sb = j & 1;   // TMEM buffer
        if (!mbar_wait(smem_u32(&kv_full[st]), (j / kBwdStages) & 1, DEV_ERR_TIMEOUT_FULL, 53) ||
            !mbar_wait(smem_u32(&s_free[sb]), ((j >> 1) & 1) ^ 1, DEV_ERR_TIMEOUT_ACC, 54)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ak = smem_u32(sm + kB_OffK + st * 2 * kBwdSub64);
        const uint32_t av = smem_u32(sm + kB_OffV + st * 2 * kBwdSub64);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t c128 = (kk >> 2) * kBwdSub128 + (kk & 3) * 32;
          const uint32_t c64 = (kk >> 2) * kBwdSub64 + (kk & 3) * 32;
          tc_mma_bf16(tmem + sb * 128, sw128_desc(aq + c128, 16, 1024), sw128_desc(ak + c64, 16, 1024),
                      IDESC_S, kk > 0 ? 1u : 0u);
          tc_mma_bf16(tmem + sb * 128 + 64, sw128_desc(ado + c128, 16, 1024),
                      sw128_desc(av + c64, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&s_full[sb]));
        if (j >= 1 && !grad(j - 1)) ok = false;
      }
      if (ok && grad(n_kt - 1)) tc_commit(smem_u32(acc_done));
    }
  } else {
    // -------------------------------------------------------------- dS (row = query)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int q = q0 + r;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    const bool q_ok = q < p.seq;
    const float lse2 = q_ok ? p.lse[stat0 + q] : INFINITY;
    // delta = rowsum(dO * O): each of the two warps of the row sums half of
    // the columns, the halves meet in shared memory.
    float dpart = 0.f;
    if (q_ok) {
      const long long off = (long long)(row_tok + q) * (p.hp * D) + lh * D;
      const uint4* o4 = reinterpret_cast<const uint4*>(p.o[part] + off);
      const uint4* d4 = reinterpret_cast<const uint4*>(p.d_o[part] + off);
      for (int c = half; c < D / 8; c += 2) {
        const uint4 a = o4[c], d = d4[c];
        dpart += bf16_lo(a.x) * bf16_lo(d.x) + bf16_hi(a.x) * bf16_hi(d.x) +
                 bf16_lo(a.y) * bf16_lo(d.y) + bf16_hi(a.y) * bf16_hi(d.y) +
                 bf16_lo(a.z) * bf16_lo(d.z) + bf16_hi(a.z) * bf16_hi(d.z) +
                 bf16_lo(a.w) * bf16_lo(d.w) + bf16_hi(a.w) * bf16_hi(d.w);
      }
    }
    float* dsum = reinterpret_cast<float*>(sm + kB_OffDelta);
    dsum[half * 128 + r] = dpart;
    named_barrier_sync(1, kBwdEwThreads);
    const float dlt = dsum[r] + dsum[128 + r];
    if (q_ok && half == 0) p.delta[stat0 + q] = dlt;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int sb = j & 1;
      if (!mbar_wait_warp(smem_u32(&s_full[sb]), (j >> 1) & 1, DEV_ERR_TIMEOUT_ACC, 55)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[32], dv[32];
      tmem_ld32x2_wait(tmem + t_lane + sb * 128 + 32 * half, sv, tmem + t_lane + sb * 128 + 64 + 32 * half,
                       dv);
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[sb]));
      const int kh = j * BK + 32 * half;                 // first key of this half
      const bool need_mask = (kh + 32 > n_valid) || (p.causal && kh + 31 > q0);
      float ds[32];
      uint32_t keep = 0xFFFFFFFFu;
      float dsc = 1.f;
      if constexpr (DROP) {
        keep = drop_keep32(p.drop, static_cast<uint32_t>((b * p.heads_total + p.head0 + head) * p.seq + q),
                           static_cast<uint32_t>(kh));
        dsc = p.drop.scale;
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float pv = ex2_approx(fmaf(__uint_as_float(sv[c]), p.scale_log2, -lse2));
        if (need_mask && (kh + c >= n_valid || (p.causal && kh + c > q))) pv = 0.f;
        ds[c] = pv * ((((keep >> c) & 1u) ? __uint_as_float(dv[c]) * dsc : 0.f) - dlt);
      }
      if (j >= 1 && !mbar_wait_warp(smem_u32(ds_free), (j - 1) & 1, DEV_ERR_TIMEOUT_ACC, 56)) {
        ok = false;
        break;
      }
      store_half_row_sw128(sm + kB_OffDS, r, half, ds);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
    }
    __nv_bfloat16* rowp = dqkv + (long long)(row_tok + q) * ldq + lh * D;
    const int nrb = (p.seq + 31) / 32;
    const int rb = (q0 + quarter * 32) / 32;   // this warp's 32-row block
    float* cs = p.colsum + ((long long)part * p.batch * nrb + b * nrb + rb) * ldq + lh * D;
    if (n_kt == 0) {
      if (q_ok && half == 0)
        for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(rowp + c) = make_uint4(0, 0, 0, 0);
      if (rb < nrb)
        for (int c = half; c < D / 32; c += 2) cs[c * 32 + lane] = 0.f;
    } else if (ok && mbar_wait_warp(smem_u32(acc_done), 0, DEV_ERR_TIMEOUT_ACC, 57)) {
      // tcgen05.ld is warp-collective: every lane loads, only valid rows store.
      // The two warps of a lane quarter take alternate 32-column chunks.
      tc_fence_after();
#pragma unroll
      for (int c = half; c < D / 32; c += 2) {
        uint32_t v[32];
        tmem_ld32_wait(tmem + t_lane + 256 + c * 32, v);
        if (q_ok) store_bf16x32(rowp + c * 32, v, p.scale);
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = q_ok ? __uint_as_float(v[e]) * p.scale : 0.f;
        warp_colsum32(f);
        if (rb < nrb) cs[c * 32 + lane] = f[0];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- fused-path helpers

// delta[b][head][q] = sum_d dO * O for every (token, head) row.  One warp per
// (token, partition): the partition's hp heads of a token are hp*D contiguous
// elements of O and of dO, read as 16-byte vectors by consecutive lanes (one
// coalesced 512-byte request per instruction); each vector's eight products
// go to a per-warp shared slot, and lanes 0..hp-1 add their head's D/8 slots
// in order.  (One thread per row read 192-byte rows with 32 scattered 16-byte
// accesses per instruction and was bound by the load unit, not by HBM.)
constexpr int kDeltaWarps = 8;
constexpr int kDeltaMaxVec = 512;   // hp*D / 8 for hp*D <= 4096

template <int D>
__global__ void __launch_bounds__(kDeltaWarps * 32) attn_delta_kernel(const AttnBwdParams p) {
  __shared__ float slot[kDeltaWarps][kDeltaMaxVec];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nparts = p.heads / p.hp;
  const long long tokens = (long long)p.batch * p.seq;
  const long long wid = (long long)blockIdx.x * kDeltaWarps + warp;
  if (wid >= tokens * nparts) return;   // warp-uniform; only warp-level sync below
  const long long tok = wid / nparts;
  const int part = static_cast<int>(wid - tok * nparts);
  const int nvec = p.hp * D / 8;
  const uint4* o4 = reinterpret_cast<const uint4*>(p.o[part] + tok * (p.hp * D));
  const uint4* d4 = reinterpret_cast<const uint4*>(p.d_o[part] + tok * (p.hp * D));
  float* sl = slot[warp];
  // The same (token, partition) row of the fp32 dQ accumulator is cleared
  // here, before the backward kernel adds into it.
  float4* z4 = reinterpret_cast<float4*>(p.dq_acc[part] + tok * (p.hp * D));
  for (int v = lane; v < p.hp * D / 4; v += 32) z4[v] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int v = lane; v < nvec; v += 32) {
    const uint4 a = o4[v], d = d4[v];
    sl[v] = ((bf16_lo(a.x) * bf16_lo(d.x) + bf16_hi(a.x) * bf16_hi(d.x)) +
             (bf16_lo(a.y) * bf16_lo(d.y) + bf16_hi(a.y) * bf16_hi(d.y))) +
            ((bf16_lo(a.z) * bf16_lo(d.z) + bf16_hi(a.z) * bf16_hi(d.z)) +
             (bf16_lo(a.w) * bf16_lo(d.w) + bf16_hi(a.w) * bf16_hi(d.w)));
  }
  __syncwarp();
  for (int lh = lane; lh < p.hp; lh += 32) {
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) acc += sl[lh * (D / 8) + c];
    const int b = static_cast<int>(tok / p.seq), q = static_cast<int>(tok - (long long)b * p.seq);
    p.delta[((long long)b * p.heads + part * p.hp + lh) * p.seq + q] = acc;
  }
}

// dQ_i = scale * accumulator -> bf16 into the Q columns of dQKV_i, and the
// column partials of those columns per 32-row block of each sequence (the
// Q part of db_qkv,i).  Block (sequence b, row block rb, partition i); each
// thread owns 4 of the hp*D columns and walks the block's rows.
template <int D>
__global__ void __launch_bounds__(128) attn_dq_convert_kernel(const AttnBwdParams p) {
  const int nrb = (p.seq + 31) / 32;
  const int b = blockIdx.x / nrb, rb = blockIdx.x % nrb;
  const int part = blockIdx.y;
  const int width = p.hp * D;
  const long long ldq = 3LL * width;
  const int r0 = rb * 32, r1 = min(p.seq, r0 + 32);
  for (int c4 = threadIdx.x; c4 < width / 4; c4 += blockDim.x) {
    float sum[4] = {0.f, 0.f, 0.f, 0.f};
    // eight rows' loads in flight at a time
    for (int r8 = r0; r8 < r1; r8 += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const long long tok = (long long)b * p.seq + r8 + u;
        v[u] = r8 + u < r1 ? __ldcs(reinterpret_cast<const float4*>(p.dq_acc[part] + tok * width) + c4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (r8 + u >= r1) break;
        const long long tok = (long long)b * p.seq + r8 + u;
        const float f[4] = {v[u].x * p.scale, v[u].y * p.scale, v[u].z * p.scale, v[u].w * p.scale};
#pragma unroll
        for (int e = 0; e < 4; ++e) sum[e] += f[e];
        reinterpret_cast<uint2*>(p.dqkv[part] + tok * ldq)[c4] =
            make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
      }
    }
    float* cs = p.colsum + ((long long)part * p.batch * nrb + (long long)b * nrb + rb) * ldq + 4 * c4;
    *reinterpret_cast<float4*>(cs) = make_float4(sum[0], sum[1], sum[2], sum[3]);
  }
}

template <int D, bool DROP>
int bwd_tc_inst(const AttnArgs& a, cudaStream_t s) {
  constexpr bool kFused = D <= 96;
  constexpr size_t kFusedSmem = FbSmem<(D + 63) / 64>::BYTES;
  static std::atomic<unsigned long long> configured{0};   // one bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    cudaError_t e;
    if constexpr (kFused) {
      e = cudaFuncSetAttribute(attn_bwd_fused_tc_kernel<D, DROP>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kFusedSmem));
    } else {
      e = cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel<D, DROP>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kA_Smem));
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<D, DROP>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kB_Smem));
    }
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const int hp = a.heads / a.t;
  const long long tokens = (long long)a.batch * a.seq;
  AttnBwdMaps maps;
  memset(&maps, 0, sizeof(maps));
  AttnBwdParams prm;
  memset(&prm, 0, sizeof(prm));
  for (int i = 0; i < a.t; ++i) {
    const long long w = 3LL * hp * D, wo = (long long)hp * D;
    if (!make_map(&maps.qkv128[i], a.qkv[i], w, tokens, w, 128) ||
        !make_map(&maps.qkv64[i], a.qkv[i], w, tokens, w, 64) ||
        !make_map(&maps.do128[i], a.d_o[i], wo, tokens, wo, 128) ||
        !make_map(&maps.do64[i], a.d_o[i], wo, tokens, wo, 64))
      return cudaErrorInvalidValue;
    prm.dqkv[i] = static_cast<__nv_bfloat16*>(a.dqkv[i]);
    if constexpr (kFused) {
      if (!a.dq_acc) return cudaErrorInvalidValue;
      prm.dq_acc[i] = a.dq_acc + (size_t)i * tokens * wo;
      if (!make_map_f32(&maps.dqacc[i], prm.dq_acc[i], wo, tokens, wo, D, 64))
        return cudaErrorInvalidValue;
    }
  }
  prm.batch = a.batch;
  prm.seq = a.seq;
  prm.heads = a.heads;
  prm.hp = hp;
  prm.causal = a.causal;
  prm.scale = 1.0f / sqrtf(static_cast<float>(D));
  prm.scale_log2 = prm.scale * kLog2e;
  prm.valid_len = a.valid_len;
  prm.lse = a.lse;
  prm.delta = a.delta;
  prm.colsum = a.colsum;
  prm.drop = a.drop;
  prm.head0 = a.head0;
  prm.heads_total = a.heads_total > 0 ? a.heads_total : a.heads;
  prm.n_sms = num_sms();
  for (int i = 0; i < a.t; ++i) {
    prm.o[i] = static_cast<const __nv_bfloat16*>(a.o[i]);
    prm.d_o[i] = static_cast<const __nv_bfloat16*>(a.d_o[i]);
  }
  const dim3 grid(a.batch * a.heads, (a.seq + 127) / 128);
  if constexpr (kFused) {
    // delta, with the fp32 dQ accumulator cleared in the same pass
    const long long dwarps = (long long)a.batch * a.seq * (a.heads / hp);
    attn_delta_kernel<D><<<static_cast<unsigned>((dwarps + kDeltaWarps - 1) / kDeltaWarps),
                           kDeltaWarps * 32, 0, s>>>(prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_bwd_fused_tc_kernel<D, DROP><<<grid, kFbThreads, kFusedSmem, s>>>(maps, prm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const dim3 cgrid(a.batch * ((a.seq + 31) / 32), a.t);
    attn_dq_convert_kernel<D><<<cgrid, 128, 0, s>>>(prm);
    return cudaGetLastError();
  } else {
    // dQ first: it also produces delta for the dK/dV kernel.
    attn_bwd_dq_tc_kernel<D, DROP><<<grid, kBwdThreads, kB_Smem, s>>>(maps, prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_bwd_dkdv_tc_kernel<D, DROP><<<grid, kBwdThreads, kA_Smem, s>>>(maps, prm);
    return cudaGetLastError();
  }
}

}  // namespace

int attention_read_clear_error(unsigned int* value) { return read_clear_unit_error(value); }

// Kernels launched by one launch_attention_bwd_tc call.
int attention_bwd_launches(int head_dim) { return head_dim <= 96 ? 3 : 2; }

namespace {

}  // namespace

int launch_attention_bwd_tc(const AttnArgs& a, cudaStream_t s) {
  const bool drop = a.drop.thresh != 0;
  switch (a.head_dim) {
    case 64: return drop ? bwd_tc_inst<64, true>(a, s) : bwd_tc_inst<64, false>(a, s);
    case 96: return drop ? bwd_tc_inst<96, true>(a, s) : bwd_tc_inst<96, false>(a, s);
    case 128: return drop ? bwd_tc_inst<128, true>(a, s) : bwd_tc_inst<128, false>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tp
