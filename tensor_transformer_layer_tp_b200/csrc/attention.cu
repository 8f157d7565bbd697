// Per-head softmax attention backward for head-split partitions (the forward
// runs on the tensor cores, attention_tc.cu).
//
// Megatron-LM splits self-attention by head: each partition computes Q, K, V
// for its own heads and runs attention locally with no communication
// (Megatron-LM show notes, the outline item on parallelising K, Q, V in the
// self-attention block; rkmt.cn guide, section 3.2).  Here a CTA owns one
// (sequence, head) pair and a tile of queries (forward) or keys (backward);
// the head's partition selects which projection buffer it reads.
//
// S = Q K^T / sqrt(d) never reaches HBM: the forward saves only
// lse = log sum exp(S) per query and the backward recomputes P = exp(S - lse)
// tile by tile.
//
// Tiles are multiplied with warp-level mma.sync (m16n8k16, bf16 in, fp32
// accumulate) from padded shared-memory tiles loaded with cp.async.
#include "kernels.cuh"
#include "tp_common.cuh"

namespace tp {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = smem_u32(smem);
  const int bytes = valid ? 16 : 0;   // 0 source bytes -> the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

// d += a * b for one m16n8k16 tile.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct PartPtrs {
  const __nv_bfloat16* qkv[8];
  __nv_bfloat16* o[8];
  const __nv_bfloat16* d_o[8];
  __nv_bfloat16* dqkv[8];
};

struct AttnGeom {
  int batch, seq, heads, hp, causal;
  float scale_log2;   // log2(e) / sqrt(d)
  float scale;        // 1 / sqrt(d)
};

__device__ __forceinline__ int valid_keys(const int32_t* valid_len, int b, int seq) {
  if (!valid_len) return seq;
  const int v = valid_len[b];
  return v < 0 ? 0 : (v > seq ? seq : v);
}

// ----------------------------------------------------------------------- backward

// delta[b, head, q] = sum_c dO[q, c] * O[q, c]; one warp per (token, head).
template <int D>
__global__ void __launch_bounds__(256) attn_delta_kernel(const __grid_constant__ PartPtrs pp,
                                                         const AttnGeom g,
                                                         float* __restrict__ delta) {
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long long total = (long long)g.batch * g.seq * g.heads;
  if (w >= total) return;
  const int head = (int)(w % g.heads);
  const long long tok = w / g.heads;
  const int part = head / g.hp, lh = head % g.hp;
  const long long ldo = (long long)g.hp * D;
  const __nv_bfloat16* o = pp.o[part] + tok * ldo + lh * D;
  const __nv_bfloat16* d_o = pp.d_o[part] + tok * ldo + lh * D;
  float s = 0.f;
  for (int c = lane * 2; c < D; c += 64) {
    const uint32_t a = *reinterpret_cast<const uint32_t*>(o + c);
    const uint32_t d = *reinterpret_cast<const uint32_t*>(d_o + c);
    s += bf16_lo(a) * bf16_lo(d) + bf16_hi(a) * bf16_hi(d);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const int b = (int)(tok / g.seq), q = (int)(tok % g.seq);
    delta[((long long)b * g.heads + head) * g.seq + q] = s;
  }
}

template <int D>
struct BwdCfg {
  static constexpr int BK = 64, BQ = 64, LDS = D + 8, LDP = 64 + 8;
  static constexpr size_t SMEM = size_t(6 * 64) * LDS * 2 + size_t(64) * LDP * 2 + 4 * 64 * 4;
};

// One CTA per (sequence, head, 64-key tile); warp w owns keys [16w, 16w+16)
// and accumulates their dK, dV in registers while walking the query tiles.
// dQ partial sums go to an fp32 scratch with atomic adds.
template <int D>
__global__ void __launch_bounds__(128) attn_bwd_kernel(const __grid_constant__ PartPtrs pp,
                                                       const AttnGeom g,
                                                       const int32_t* __restrict__ valid_len,
                                                       const float* __restrict__ lse,
                                                       const float* __restrict__ delta,
                                                       float* __restrict__ dq_acc) {
  using C = BwdCfg<D>;
  constexpr int BK = C::BK, BQ = C::BQ, LDS = C::LDS, LDP = C::LDP;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sV = sK + BK * LDS;
  __nv_bfloat16* sQ = sV + BK * LDS;        // [2][BQ][LDS]
  __nv_bfloat16* sdO = sQ + 2 * BQ * LDS;   // [2][BQ][LDS]
  __nv_bfloat16* sdS = sdO + 2 * BQ * LDS;  // [BQ][LDP]  dS[query][key]
  float* sL = reinterpret_cast<float*>(sdS + BQ * LDP);   // [2][BQ] lse * log2(e)
  float* sD = sL + 2 * BQ;                                 // [2][BQ] delta

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int b = blockIdx.y / g.heads, head = blockIdx.y % g.heads;
  const int part = head / g.hp, lh = head % g.hp;
  const long long ld = 3LL * g.hp * D;
  const long long ldo = (long long)g.hp * D;
  const long long row0 = (long long)b * g.seq;
  const int k0 = blockIdx.x * BK;
  const int n_valid = valid_keys(valid_len, b, g.seq);
  const __nv_bfloat16* qkv = pp.qkv[part];
  const __nv_bfloat16* d_o = pp.d_o[part];
  __nv_bfloat16* dqkv = pp.dqkv[part];
  const long long stat0 = ((long long)b * g.heads + head) * g.seq;

  const int key_w = k0 + warp * 16;   // first key of this warp
  if (k0 >= n_valid) {
    // Every key of the tile is padding: its gradients are zero.
    for (int c = tid; c < BK * D / 2; c += 128) {
      const int r = c / (D / 2), cc = (c % (D / 2)) * 2;
      if (k0 + r < g.seq) {
        __nv_bfloat16* rowp = dqkv + (row0 + k0 + r) * ld;
        *reinterpret_cast<uint32_t*>(rowp + g.hp * D + lh * D + cc) = 0u;
        *reinterpret_cast<uint32_t*>(rowp + 2 * g.hp * D + lh * D + cc) = 0u;
      }
    }
    return;
  }

  constexpr int CH = D / 8;
  for (int c = tid; c < BK * CH; c += 128) {
    const int r = c / CH, cc = c - r * CH;
    const int pos = k0 + r;
    const bool ok = pos < g.seq;
    const __nv_bfloat16* base = qkv + (row0 + (ok ? pos : 0)) * ld + cc * 8;
    cp_async16(sK + r * LDS + cc * 8, base + (long long)g.hp * D + lh * D, ok);
    cp_async16(sV + r * LDS + cc * 8, base + 2LL * g.hp * D + lh * D, ok);
  }
  const int q_begin = g.causal ? (k0 / BQ) * BQ : 0;
  const int n_qt = (g.seq - q_begin + BQ - 1) / BQ;
  auto load_q = [&](int it, int buf) {
    const int q0 = q_begin + it * BQ;
    for (int c = tid; c < BQ * CH; c += 128) {
      const int r = c / CH, cc = c - r * CH;
      const int pos = q0 + r;
      const bool ok = pos < g.seq;
      const long long tok = row0 + (ok ? pos : 0);
      cp_async16(sQ + (buf * BQ + r) * LDS + cc * 8, qkv + tok * ld + lh * D + cc * 8, ok);
      cp_async16(sdO + (buf * BQ + r) * LDS + cc * 8, d_o + tok * ldo + lh * D + cc * 8, ok);
    }
    if (tid < BQ) {
      const int pos = q0 + tid;
      const bool ok = pos < g.seq;
      sL[buf * BQ + tid] = ok ? lse[stat0 + pos] * kLog2e : INFINITY;
      sD[buf * BQ + tid] = ok ? delta[stat0 + pos] : 0.f;
    }
  };
  load_q(0, 0);
  cp_async_commit();

  float acc_dk[D / 8][4], acc_dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc_dk[i][e] = acc_dv[i][e] = 0.f;

  for (int it = 0; it < n_qt; ++it) {
    const int buf = it & 1;
    const int q0 = q_begin + it * BQ;
    if (it + 1 < n_qt) {
      load_q(it + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* bQ = sQ + buf * BQ * LDS;
    const __nv_bfloat16* bdO = sdO + buf * BQ * LDS;
    const float* bL = sL + buf * BQ;
    const float* bD = sD + buf * BQ;

    // S^T = K_w Q^T  (16 keys x 64 queries)
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t kf[4];
      ldsm_x4(sK + (warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + ks * 16 + (lane >> 4) * 8,
              kf[0], kf[1], kf[2], kf[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        // B fragments for query n-tiles 2np, 2np+1 at this k-step
        uint32_t b0, b1, b2, b3;
        ldsm_x4(bQ + (np * 16 + (lane & 7) + (lane >> 4) * 8) * LDS + ks * 16 + ((lane >> 3) & 1) * 8,
                b0, b1, b2, b3);
        mma16816(s[2 * np], kf, b0, b1);
        mma16816(s[2 * np + 1], kf, b2, b3);
      }
    }
    // P^T = exp(S^T * scale - lse[query]) with masks.
    const bool need_mask = (g.causal && q0 < key_w + 16) || (k0 + BK > n_valid);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int qc = nt * 8 + 2 * tig + (i & 1);
        float p = exp2f(s[nt][i] * g.scale_log2 - bL[qc]);
        if (need_mask) {
          const int key = key_w + gid + (i >> 1) * 8;
          const int qry = q0 + qc;
          if (key >= n_valid || (g.causal && qry < key)) p = 0.f;
        }
        s[nt][i] = p;
      }
    }
    // dV_w += P^T dO
    {
      uint32_t pf[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        pf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(s[nt][0], s[nt][1]);
        pf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(s[nt][2], s[nt][3]);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
        for (int nd = 0; nd < D / 16; ++nd) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(bdO + (ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + nd * 16 +
                        (lane >> 4) * 8,
                    b0, b1, b2, b3);
          mma16816(acc_dv[2 * nd], pf[ks], b0, b1);
          mma16816(acc_dv[2 * nd + 1], pf[ks], b2, b3);
        }
      }
    }
    // dP^T = V_w dO^T ; dS^T = P^T * (dP^T - delta[query])
    float dp[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) dp[nt][0] = dp[nt][1] = dp[nt][2] = dp[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t vf[4];
      ldsm_x4(sV + (warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + ks * 16 + (lane >> 4) * 8,
              vf[0], vf[1], vf[2], vf[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(bdO + (np * 16 + (lane & 7) + (lane >> 4) * 8) * LDS + ks * 16 + ((lane >> 3) & 1) * 8,
                b0, b1, b2, b3);
        mma16816(dp[2 * np], vf, b0, b1);
        mma16816(dp[2 * np + 1], vf, b2, b3);
      }
    }
    uint32_t dsf[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float ds[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int qc = nt * 8 + 2 * tig + (i & 1);
        ds[i] = s[nt][i] * (dp[nt][i] - bD[qc]);
      }
      dsf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(ds[0], ds[1]);
      dsf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(ds[2], ds[3]);
      // dS[query][key] for the dQ product below
      const int kr = warp * 16 + gid;
      const int qc = nt * 8 + 2 * tig;
      sdS[(qc + 0) * LDP + kr] = __float2bfloat16_rn(ds[0]);
      sdS[(qc + 1) * LDP + kr] = __float2bfloat16_rn(ds[1]);
      sdS[(qc + 0) * LDP + kr + 8] = __float2bfloat16_rn(ds[2]);
      sdS[(qc + 1) * LDP + kr + 8] = __float2bfloat16_rn(ds[3]);
    }
    // dK_w += dS^T Q
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int nd = 0; nd < D / 16; ++nd) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(bQ + (ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + nd * 16 +
                      (lane >> 4) * 8,
                  b0, b1, b2, b3);
        mma16816(acc_dk[2 * nd], dsf[ks], b0, b1);
        mma16816(acc_dk[2 * nd + 1], dsf[ks], b2, b3);
      }
    }
    __syncthreads();
    // dQ[16 queries of this warp] += dS K, accumulated into fp32 scratch.
    {
      uint32_t af[4][4];
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ldsm_x4(sdS + (warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDP + ks * 16 + (lane >> 4) * 8,
                af[ks][0], af[ks][1], af[ks][2], af[ks][3]);
      float* dq = dq_acc + ((long long)part * g.batch * g.seq + row0) * ldo + lh * D;
#pragma unroll
      for (int chunk = 0; chunk < D / 32; ++chunk) {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
          for (int nd = 0; nd < 2; ++nd) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sK + (ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + chunk * 32 +
                          nd * 16 + (lane >> 4) * 8,
                      b0, b1, b2, b3);
            mma16816(acc[2 * nd], af[ks], b0, b1);
            mma16816(acc[2 * nd + 1], af[ks], b2, b3);
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int q = q0 + warp * 16 + gid + r * 8;
          if (q < g.seq) {
            float* rowp = dq + (long long)q * ldo + chunk * 32 + 2 * tig;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
              atomicAdd(reinterpret_cast<float2*>(rowp + nt * 8),
                        make_float2(acc[nt][2 * r] * g.scale, acc[nt][2 * r + 1] * g.scale));
          }
        }
      }
    }
  }

  // dK = scale * dS^T Q, dV = P^T dO for this warp's 16 keys.
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int key = key_w + gid + r * 8;
    if (key < g.seq) {
      __nv_bfloat16* rowp = dqkv + (row0 + key) * ld;
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        const int c = nt * 8 + 2 * tig;
        *reinterpret_cast<uint32_t*>(rowp + g.hp * D + lh * D + c) =
            pack_bf16(acc_dk[nt][2 * r] * g.scale, acc_dk[nt][2 * r + 1] * g.scale);
        *reinterpret_cast<uint32_t*>(rowp + 2 * g.hp * D + lh * D + c) =
            pack_bf16(acc_dv[nt][2 * r], acc_dv[nt][2 * r + 1]);
      }
    }
  }
}

// dQ section of dqkv = bf16(dq_acc); 8 elements per thread.
__global__ void __launch_bounds__(256) attn_dq_convert_kernel(const __grid_constant__ PartPtrs pp,
                                                              int t, long long tokens, int hp_d,
                                                              const float* __restrict__ dq_acc) {
  const long long per_part = tokens * (hp_d / 8);
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= per_part * t) return;
  const int part = (int)(idx / per_part);
  const long long rem = idx - part * per_part;
  const long long tok = rem / (hp_d / 8);
  const int c = (int)(rem % (hp_d / 8)) * 8;
  const float4* src = reinterpret_cast<const float4*>(dq_acc + ((long long)part * tokens + tok) * hp_d + c);
  const float4 a = src[0], b = src[1];
  uint4 o = make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
  *reinterpret_cast<uint4*>(pp.dqkv[part] + tok * 3LL * hp_d + c) = o;
}

PartPtrs make_parts(const AttnArgs& a) {
  PartPtrs p;
  for (int i = 0; i < 8; ++i) {
    const bool in = i < a.t;
    p.qkv[i] = in ? static_cast<const __nv_bfloat16*>(a.qkv[i]) : nullptr;
    p.o[i] = in ? static_cast<__nv_bfloat16*>(a.o[i]) : nullptr;
    p.d_o[i] = in ? static_cast<const __nv_bfloat16*>(a.d_o[i]) : nullptr;
    p.dqkv[i] = in ? static_cast<__nv_bfloat16*>(a.dqkv[i]) : nullptr;
  }
  return p;
}

AttnGeom make_geom(const AttnArgs& a) {
  AttnGeom g;
  g.batch = a.batch;
  g.seq = a.seq;
  g.heads = a.heads;
  g.hp = a.heads / a.t;
  g.causal = a.causal;
  g.scale = 1.0f / sqrtf(static_cast<float>(a.head_dim));
  g.scale_log2 = g.scale * kLog2e;
  return g;
}

template <int D>
int bwd_inst(const AttnArgs& a, cudaStream_t s) {
  using C = BwdCfg<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const PartPtrs pp = make_parts(a);
  const AttnGeom g = make_geom(a);
  const long long tokens = (long long)a.batch * a.seq;
  const int hp_d = (a.heads / a.t) * D;
  cudaError_t e = cudaMemsetAsync(a.dq_acc, 0, sizeof(float) * tokens * hp_d * a.t, s);
  if (e != cudaSuccess) return e;
  const long long warps = tokens * a.heads;
  attn_delta_kernel<D><<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(pp, g, a.delta);
  dim3 grid((a.seq + C::BK - 1) / C::BK, a.batch * a.heads);
  attn_bwd_kernel<D><<<grid, 128, C::SMEM, s>>>(pp, g, a.valid_len, a.lse, a.delta, a.dq_acc);
  const long long n8 = tokens * (hp_d / 8) * a.t;
  attn_dq_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(pp, a.t, tokens, hp_d,
                                                                     a.dq_acc);
  return cudaGetLastError();
}

}  // namespace

int launch_attention_delta(const AttnArgs& a, cudaStream_t s) {
  const PartPtrs pp = make_parts(a);
  const AttnGeom g = make_geom(a);
  const long long warps = (long long)a.batch * a.seq * a.heads;
  const unsigned blocks = (unsigned)((warps + 7) / 8);
  switch (a.head_dim) {
    case 64: attn_delta_kernel<64><<<blocks, 256, 0, s>>>(pp, g, a.delta); break;
    case 96: attn_delta_kernel<96><<<blocks, 256, 0, s>>>(pp, g, a.delta); break;
    case 128: attn_delta_kernel<128><<<blocks, 256, 0, s>>>(pp, g, a.delta); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int launch_attention_bwd(const AttnArgs& a, cudaStream_t s) {
  switch (a.head_dim) {
    case 64: return bwd_inst<64>(a, s);
    case 96: return bwd_inst<96>(a, s);
    case 128: return bwd_inst<128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tp
