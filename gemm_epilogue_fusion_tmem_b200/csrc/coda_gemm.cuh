// Persistent, warp-specialised tcgen05 GEMM with fused epilogues (sm_100a).
//
// GEMM-epilogue structure (toolin.ai CODA article, section 核心の洞察; kucoin.com
// (ru) CODA article, section «В «Финале» спрятаны сокровища»): a fixed mainloop
// computes an fp32 tile into tensor memory, and an epilogue transforms the
// tile while it is still on chip before anything reaches HBM.  The epilogue
// variants are built from the pages' primitives (five-primitive table):
// elementwise transforms (residual add, SwiGLU, its backward, RoPE), vector
// loads (r, c, g), matrix-tile loads/stores (R, H, a/b, outputs), tile-wise
// reductions (row sums of squares, column sums for dg) and, for the
// cross-entropy, the stateful online max / sum-exp.
//
// Tiles: by default a CTA pair (cluster of 2, tcgen05 cta_group::2) computes a
// 256 x 256 tile, each CTA holding 128 rows of A and half of B; with PAIR =
// false one CTA computes 128 x 256.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer (one lane): 128B-swizzled K-major or MN-major
//               operand tiles into a STAGES-deep shared-memory ring.
//   warp 1      TMEM owner and MMA issuer (one lane of the pair's leader):
//               tcgen05.mma kind::f16, K=16, into one of two TMEM
//               accumulators (2 x 256 columns), commits -> mbarriers.
//   warps 2-5   epilogue: tcgen05.ld 32 lanes x 32 columns per step, one
//               output row per thread; outputs staged in shared memory and
//               written with TMA tile stores.
// The two TMEM accumulators let tile i's epilogue overlap tile i+1's mainloop.
// Every wait is bounded (see mbar_wait); a role that gives up records the
// failure in the status word and the CTA drains and exits.
#pragma once

#include "coda_ptx.cuh"

namespace coda {

constexpr int BM = 128;              // tile rows (TMEM lanes)
constexpr int BN = 256;              // tile columns (TMEM columns per accumulator)
constexpr int BK = 64;               // reduction depth per stage (128 bytes of bf16)
constexpr int UMMA_K = 16;
constexpr int MN_CHUNK_BYTES = 64 * BK * 2;  // one [64 k][64 mn] MN-major chunk, 8 KiB
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;

enum Epi : int {
  EPI_STORE = 0,       // out = bf16(acc [* g_col])
  EPI_RESID_RMS = 1,   // H = bf16(acc + R); P[row, ntile] = sum H^2; optional Hg = bf16(H*g) (H the stored bf16)
  EPI_SWIGLU = 2,      // a = r*acc_gate, b = r*acc_up; Y = silu(a)*b; AB = [a|b]
  EPI_DN = 3,          // dH = g*acc - c*H (+dH_in); column partials of acc*H
  EPI_SWIGLU_BWD = 4,  // dY = acc; da, db from a, b; dA = [da|db] (optionally r-scaled, with c partials)
  EPI_XENT = 5,        // logits tile: per-row online (max, sum exp) partials + the target logit
  EPI_XENT_BWD = 6,    // dlogits = dloss_i (exp(logit - lse_i) - [j == t_i]), stored bf16
  EPI_ROPE = 7,        // QKV tile: rotate the q/k heads' (j, j + hd/2) pairs by pos * base^(-2j/hd)
};

struct GemmParams {
  int M;            // output rows
  int N;            // output columns (EPI_SWIGLU / EPI_SWIGLU_BWD: F)
  int K;            // reduction length
  int num_m_tiles;
  int num_n_tiles;
  int k_blocks;
  int group_m;      // rasterisation (see tile_coords): >0 row-tile groups, <0 column-tile groups
  int split;        // EPI_SWIGLU: row offset of the up half in B and column offset of b in AB;
                    // EPI_SWIGLU_BWD: column offset of b / db (= F)
  __nv_bfloat16* out;
  int ldo;
  const __nv_bfloat16* in0;  // R (RESID_RMS), H (DN), AB (SWIGLU_BWD)
  int ld_in0;
  const __nv_bfloat16* in1;  // dH_in (DN), optional
  const __nv_bfloat16* colvec;  // g (STORE scale, DN), optional for STORE
  const float* rowvec;          // r (SWIGLU, optional), c (DN)
  float* part;                  // P (RESID_RMS; read by SWIGLU to form r), Pg (DN)
  int ld_part;
  __nv_bfloat16* out2;          // AB (SWIGLU), Hg (RESID_RMS), optional
  int ldo2;
  const int* tgt;               // target class per row (XENT, XENT_BWD)
  const float* rowvec2;         // dloss (XENT_BWD)
  float* outf;                  // target logit per row (XENT); r (SWIGLU with part)
  int head_dim;                 // ROPE: head width (64, 128 or 256)
  int rot_cols;                 // ROPE: columns [0, rot_cols) are rotated (q and k heads)
  int seq_len;                  // ROPE: position = row % seq_len
  float rope_k;                 // ROPE: -2 log2(base) / head_dim, so inv_freq_j = 2^(j * rope_k)
  float inv_d;                  // SWIGLU with part: 1 / d of the RMSNorm mean
  float eps;                    // SWIGLU with part: the RMSNorm eps
  uint32_t* status;
  unsigned long long wait_limit_ns;
  uint32_t kernel_id;
};

// Tile order.  group > 0: groups of `group` row tiles, the row tile varying
// fastest inside a group, so the group's A rows stay in L2 while B streams
// through.  group < 0: the same with the roles of rows and columns swapped
// (groups of -group column tiles, column tile fastest).
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group, int& m_blk, int& n_blk) {
  if (group > 0) {
    const int group_size = group * num_n;
    const int g = tile / group_size;
    const int first_m = g * group;
    const int gm = min(num_m - first_m, group);
    const int local = tile - g * group_size;
    m_blk = first_m + local % gm;
    n_blk = local / gm;
  } else {
    const int gsz = -group;
    const int group_size = gsz * num_m;
    const int g = tile / group_size;
    const int first_n = g * gsz;
    const int gn = min(num_n - first_n, gsz);
    const int local = tile - g * group_size;
    n_blk = first_n + local % gn;
    m_blk = local / gn;
  }
}

// Load 32 bf16 starting at p (16-byte aligned) as floats; zeros when !valid.
__device__ __forceinline__ void load32_bf16(const __nv_bfloat16* p, bool valid, float (&f)[32]) {
  if (valid) {
    uint4 q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = ldg_nc_v4(p + 8 * j);
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack8(q[j], f + 8 * j);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) f[i] = 0.f;
  }
}

// One thread's 32 bf16 of a row-major input chunk, held packed in registers
// so it can be loaded one chunk ahead of its use (and, for a tile's first
// chunk, before the accumulator is ready): the epilogue's per-row inputs
// (residual, H, dH_in, saved a/b) then arrive while earlier work runs.
struct Pref32 {
  uint4 q[4];
};
__device__ __forceinline__ void pref_load(Pref32& x, const __nv_bfloat16* p, bool valid) {
#pragma unroll
  for (int j = 0; j < 4; ++j) x.q[j] = valid ? ldg_nc_v4(p + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
}
__device__ __forceinline__ void pref_unpack(const Pref32& x, float (&f)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) unpack8(x.q[j], f + 8 * j);
}

// Per-warp tile store through shared memory: the warp's 32 rows x 32 columns
// of one output go to a 2 KiB staging tile (64-byte rows, 16-byte chunks
// swizzled by (row >> 1) & 3, which makes the row-per-thread writes
// bank-conflict free and matches the tensor map's 64-byte swizzle); one lane
// then issues a TMA bulk tensor store with an evict-first L2 policy (the
// kernel never reads its outputs back; in a same-box A/B this cut the 70B
// step's DRAM traffic by 4 %).  TMA clips rows and columns outside the
// tensor, so ragged row tiles need no masking.  Up to kEpiTiles tiles per
// 32-column step.  A step that stages one tile rotates over the kEpiTiles
// slots, so it waits only for the store issued kEpiTiles steps earlier; a step
// that stages more waits until the previous step's stores have been read.
// Each output tile starts with all slots free (begin_tile), so a warp whose
// rows lie past M in one tile (it stages but stores nothing) cannot overwrite
// a slot that an earlier tile's store is still reading.
constexpr int kEpiTiles = 3;
constexpr int kEpiTileBytes = 32 * 32 * 2;
constexpr int kEpiWarpBytes = kEpiTiles * kEpiTileBytes;

struct EpiStore {
  uint8_t* stg;   // this warp's staging (kEpiWarpBytes, 1024-byte aligned)
  int lane;
  int row0;       // first output row of this warp
  int rows;       // output rows (M); a warp wholly past them stores nothing
  int n;          // tiles staged in the current step
  int base;       // first slot of the current step
  int slot;       // next slot of a one-tile step
  const CUtensorMap* map[kEpiTiles];
  int col[kEpiTiles];

  __device__ __forceinline__ void begin_tile() {
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
    slot = 0;
  }
  // Reserve the slots of one step that stages `tiles` output tiles.
  __device__ __forceinline__ void begin(int tiles = kEpiTiles) {
    static_assert(kEpiTiles == 3, "the rotating wait below allows kEpiTiles - 1 = 2 groups in flight");
    if (tiles == 1) {
      if (lane == 0) bulk_wait_read_2();
      base = slot;
      slot = (slot + 1 == kEpiTiles) ? 0 : slot + 1;
    } else {
      if (lane == 0) bulk_wait_read_all();
      base = 0;
    }
    __syncwarp();
    n = 0;
  }
  __device__ __forceinline__ void put_packed(const uint4 (&q)[4], const CUtensorMap* m, int c) {
    uint8_t* t = stg + (base + n) * kEpiTileBytes + lane * 64;
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a = smem_u32(t + ((j ^ sw) << 4));
      asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(q[j].x), "r"(q[j].y), "r"(q[j].z),
                   "r"(q[j].w)
                   : "memory");
    }
    map[n] = m;
    col[n] = c;
    ++n;
  }
  __device__ __forceinline__ void put(const float (&f)[32], const CUtensorMap* m, int c) {
    uint4 q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = pack8(f + 8 * j);
    put_packed(q, m, c);
  }
  __device__ __forceinline__ void flush() {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row0 < rows) {
      const uint64_t evict_first = l2_policy_evict_first();
      for (int t = 0; t < n; ++t)
        tma_store_2d_hint(map[t], stg + (base + t) * kEpiTileBytes, col[t], row0, evict_first);
      bulk_commit_group();
    }
  }
  __device__ __forceinline__ void finish() {
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
};

// Sum of a 32 x 32 block held one row per lane, reduced over the lanes:
// afterwards v[0] of lane l holds the sum over all lanes of column l.
// Recursive halving: 16 + 8 + 4 + 2 + 1 shuffles for 32 columns.
__device__ __forceinline__ void warp_column_sums(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
}


// The RMSNorm row scale for the gate/up GEMM: with GEMM1's partial sums of
// squares (p.part) it is formed here, r_i = 1/sqrt(sum_t P[i,t] / d + eps),
// the partials summed in column-tile order, and the row's first column tile
// stores it; otherwise it is read from p.rowvec (1 when there is none).
__device__ __forceinline__ float swiglu_row_scale(const GemmParams& p, int row, bool rv, int n_blk) {
  if (p.part == nullptr) return (p.rowvec != nullptr) ? (rv ? p.rowvec[row] : 0.f) : 1.f;
  if (!rv) return 0.f;
  const float* pr = p.part + (size_t)row * p.ld_part;
  float s = 0.f;
  for (int t = 0; t < p.ld_part; ++t) s += pr[t];
  const float r = rsqrtf(fmaf(s, p.inv_d, p.eps));
  if (n_blk == 0) p.outf[row] = r;
  return r;
}

// Loads the first chunk of a tile's per-row epilogue inputs, and the gate/up
// GEMM's row scale (issued before the wait for the accumulator).
template <int EPI>
__device__ __forceinline__ void epilogue_prefetch(const GemmParams& p, int row, bool rv, int n_blk, Pref32& x0,
                                                  Pref32& x1, float& rr) {
  if constexpr (EPI == EPI_SWIGLU) {
    rr = swiglu_row_scale(p, row, rv, n_blk);
  } else if constexpr (EPI == EPI_RESID_RMS || EPI == EPI_DN) {
    const size_t off = (size_t)row * p.ld_in0 + (size_t)n_blk * BN;
    pref_load(x0, p.in0 + off, rv);
    if constexpr (EPI == EPI_DN) {
      if (p.in1 != nullptr) pref_load(x1, p.in1 + (size_t)row * p.ldo + (size_t)n_blk * BN, rv);
    }
  } else if constexpr (EPI == EPI_SWIGLU_BWD) {
    const __nv_bfloat16* ab = p.in0 + (size_t)row * p.ld_in0 + (size_t)n_blk * BN;
    pref_load(x0, ab, rv);
    pref_load(x1, ab + p.split, rv);
  }
}

// One 128-row half-tile of the epilogue: this thread owns output row `row`
// (valid when rv), `group32` = (row - lane) / 32 indexes the per-warp partials.
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, uint32_t tbase, int row, bool rv, int group32,
                                              int n_blk, int lane, EpiStore& es, const CUtensorMap* mo1,
                                              const CUtensorMap* mo2, Pref32& x0, Pref32& x1, float rr) {
  if constexpr (EPI == EPI_STORE) {
    const int n0 = n_blk * BN;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= p.N) break;
      float v[32];
      tmem_ld32(tbase + c, v);
      if (p.colvec != nullptr) {
        float g[32];
        load32_bf16(p.colvec + n0 + c, true, g);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= g[i];
      }
      es.begin(1);
      es.put(v, mo1, n0 + c);
      es.flush();
    }
  } else if constexpr (EPI == EPI_RESID_RMS) {
    const int n0 = n_blk * BN;
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= p.N) break;
      float rres[32];
      pref_unpack(x0, rres);
      if (c + 32 < BN && n0 + c + 32 < p.N) pref_load(x0, p.in0 + (size_t)row * p.ld_in0 + n0 + c + 32, rv);
      float v[32];
      tmem_ld32(tbase + c, v);
      uint4 hq[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = v[8 * j + i] + rres[8 * j + i];
        hq[j] = pack8(h);
        unpack8(hq[j], v + 8 * j);  // v now holds the stored (bf16-rounded) H
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(v[8 * j + i], v[8 * j + i], ss);
      }
      es.begin(p.out2 != nullptr ? 2 : 1);
      es.put_packed(hq, mo1, n0 + c);
      if (p.out2 != nullptr) {
        // Activation-side gain: Hg = bf16(H * g) from the stored H, the second
        // GEMM's operand (the product of two bf16 values is exact in fp32, so
        // the only rounding is the final one).
        float g[32];
        load32_bf16(p.colvec + n0 + c, true, g);
#pragma unroll
        for (int i = 0; i < 32; ++i) g[i] *= v[i];
        es.put(g, mo2, n0 + c);
      }
      es.flush();
    }
    if (rv && p.part != nullptr) p.part[(size_t)row * p.ld_part + n_blk] = ss;
  } else if constexpr (EPI == EPI_SWIGLU) {
    constexpr int HALF = BN / 2;
    const int n0 = n_blk * HALF;
#pragma unroll 1
    for (int c = 0; c < HALF; c += 32) {
      if (n0 + c >= p.N) break;
      float a[32], b[32];
      tmem_ld32(tbase + c, a);
      tmem_ld32(tbase + HALF + c, b);
      float y[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        a[i] *= rr;
        b[i] *= rr;
        y[i] = a[i] * sigmoid_f(a[i]) * b[i];
      }
      es.begin(p.out2 != nullptr ? 3 : 1);
      es.put(y, mo1, n0 + c);
      if (p.out2 != nullptr) {
        es.put(a, mo2, n0 + c);
        es.put(b, mo2, p.split + n0 + c);
      }
      es.flush();
    }
  } else if constexpr (EPI == EPI_DN) {
    const int n0 = n_blk * BN;
    const float cc = rv ? p.rowvec[row] : 0.f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= p.N) break;
      const bool more = c + 32 < BN && n0 + c + 32 < p.N;
      float h[32];
      pref_unpack(x0, h);
      if (more) pref_load(x0, p.in0 + (size_t)row * p.ld_in0 + n0 + c + 32, rv);
      float v[32];
      tmem_ld32(tbase + c, v);
      float g[32];
      load32_bf16(p.colvec + n0 + c, true, g);
      float o[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = fmaf(g[i], v[i], -cc * h[i]);
      if (p.in1 != nullptr) {
        float e[32];
        pref_unpack(x1, e);
        if (more) pref_load(x1, p.in1 + (size_t)row * p.ldo + n0 + c + 32, rv);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] += e[i];
      }
      es.begin(1);
      es.put(o, mo1, n0 + c);
      es.flush();
      // dg partial: sum over this warp's 32 rows of acc * H, per column.
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= h[i];
      warp_column_sums(v, lane);
      p.part[(size_t)group32 * p.ld_part + n0 + c + lane] = v[0];
    }
  } else if constexpr (EPI == EPI_XENT) {
    // Stateful transform (online max / sum-exp) over this tile's columns.
    const int n0 = n_blk * BN;
    const int t = rv ? p.tgt[row] : -1;
    float m = -INFINITY, sum = 0.f, tl = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= p.N) break;
      float v[32];
      tmem_ld32(tbase + c, v);
      float cm = v[0];
#pragma unroll
      for (int i = 1; i < 32; ++i) cm = fmaxf(cm, v[i]);
      const float nm = fmaxf(m, cm);
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) acc += __expf(v[i] - nm);
      sum = sum * __expf(m - nm) + acc;
      m = nm;
      const int off = t - (n0 + c);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i == off) tl = v[i];
    }
    if (rv) {
      reinterpret_cast<float2*>(p.part)[(size_t)row * p.ld_part + n_blk] = make_float2(m, sum);
      if (t >= n0 && t < n0 + BN && t < p.N) p.outf[row] = tl;
    }
  } else if constexpr (EPI == EPI_XENT_BWD) {
    const int n0 = n_blk * BN;
    const int t = rv ? p.tgt[row] : -1;
    const float lse = rv ? p.rowvec[row] : 0.f;
    const float dl = rv ? p.rowvec2[row] : 0.f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= p.N) break;
      float v[32];
      tmem_ld32(tbase + c, v);
      const int off = t - (n0 + c);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float g = __expf(v[i] - lse);
        if (i == off) g -= 1.f;
        v[i] = g * dl;
      }
      es.begin(1);
      es.put(v, mo1, n0 + c);
      es.flush();
    }
  } else if constexpr (EPI == EPI_ROPE) {
    // Every head of the tile turns its (j, j + hd/2) pairs by the same angles
    // pos * inv_freq_j, so the sines and cosines of each 32-frequency slice
    // are computed once per row and applied to all the tile's rotated heads
    // (heads run q, k, v, so if the tile's first head is not rotated, none is).
    const int n0 = n_blk * BN;
    const float pos = (float)(row % p.seq_len);
    const int half = p.head_dim / 2;
    const bool any_rot = n0 < p.rot_cols;
#pragma unroll 1
    for (int c = 0; c < half; c += 32) {
      float sn[32], cs[32];
      if (any_rot) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sincosf(pos * exp2f((float)(c + i) * p.rope_k), &sn[i], &cs[i]);
      }
#pragma unroll 1
      for (int h0 = 0; h0 < BN; h0 += p.head_dim) {
        const int col0 = n0 + h0;
        if (col0 >= p.N) break;
        float x1[32], x2[32];
        tmem_ld32(tbase + h0 + c, x1);
        tmem_ld32(tbase + h0 + half + c, x2);
        if (col0 < p.rot_cols) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float y1 = x1[i] * cs[i] - x2[i] * sn[i];
            const float y2 = x2[i] * cs[i] + x1[i] * sn[i];
            x1[i] = y1;
            x2[i] = y2;
          }
        }
        es.begin();
        es.put(x1, mo1, col0 + c);
        es.put(x2, mo1, col0 + half + c);
        es.flush();
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU_BWD) {
    // dA = [da | db] from dY = acc and the saved a, b.  With a row scale r
    // (rowvec) the stored operand is r_i [da | db] and the tile also emits the
    // row partial sum_c (da a + db b) of the RMSNorm backward's coefficient.
    const int n0 = n_blk * BN;
    const float rr = (p.rowvec != nullptr) ? (rv ? p.rowvec[row] : 0.f) : 1.f;
    float cpart = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= p.N) break;
      float a[32], b[32];
      pref_unpack(x0, a);
      pref_unpack(x1, b);
      if (c + 32 < BN && n0 + c + 32 < p.N) {
        const __nv_bfloat16* ab = p.in0 + (size_t)row * p.ld_in0 + n0 + c + 32;
        pref_load(x0, ab, rv);
        pref_load(x1, ab + p.split, rv);
      }
      float dy[32];
      tmem_ld32(tbase + c, dy);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float s = sigmoid_f(a[i]);
        const float da = dy[i] * b[i] * s * (1.f + a[i] * (1.f - s));
        const float db = dy[i] * a[i] * s;
        cpart = fmaf(da, a[i], cpart);
        cpart = fmaf(db, b[i], cpart);
        a[i] = da * rr;
        b[i] = db * rr;
      }
      es.begin();
      es.put(a, mo1, n0 + c);
      es.put(b, mo1, p.split + n0 + c);
      es.flush();
    }
    if (rv && p.part != nullptr) p.part[(size_t)row * p.ld_part + n_blk] = cpart;
  }
}

// Per-mode constants.  PAIR = one 256 x 256 tile per CTA pair (cta_group::2:
// each CTA holds 128 rows of A and half of B, the leader issues M=256 MMAs);
// otherwise one 128 x 256 tile per CTA.
template <bool PAIR>
struct TileCfg {
  static constexpr int STAGES = PAIR ? 6 : 4;
  static constexpr int TILE_M = PAIR ? 256 : 128;
  static constexpr int B_ROWS = PAIR ? 128 : 256;      // B rows (output columns) held per CTA
  static constexpr int A_BYTES = 128 * BK * 2;         // 16 KiB
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = 4 * kEpiWarpBytes;   // staging for the 4 epilogue warps
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 256;
  static constexpr int MMA_M = PAIR ? 256 : 128;
  static constexpr int CTAS = PAIR ? 2 : 1;
};

template <int EPI, bool A_MN, bool B_MN, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO1, const __grid_constant__ CUtensorMap tmO2,
                   const GemmParams p) {
  using C = TileCfg<PAIR>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * C::A_BYTES;
  uint8_t* sEpi = sB + S * C::B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::EPI_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = the pair's leader
  const int first_tile = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
  const int tile_step = PAIR ? (int)num_clusters_x() : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4 * C::CTAS);  // one arrival per epilogue warp of the pair
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);  // same warp and slot in both CTAs
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The set-up above overlaps the previous kernel's tail; global memory is
  // touched only after it has completed.  The next kernel may start its own
  // set-up as soon as SMs free up.
  griddep_wait();
  griddep_launch_dependents();

  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns, p.kernel_id};
  const int num_tiles = p.num_m_tiles * p.num_n_tiles;
  int issued = 0;  // TMA stages issued by the producer lane

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer (every CTA)
      // Normal L2 priority for both operands: concurrent tiles of a wave reuse
      // each other's lines, which evict-first / evict-last hints were measured to
      // break (DRAM reads per launch more than doubled).
      const uint64_t hint_a = l2_policy_evict_normal();
      const uint64_t hint_b = hint_a;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = first_tile; tile < num_tiles && ok; tile += tile_step) {
        int m_blk, n_blk;
        tile_coords(tile, p.num_m_tiles, p.num_n_tiles, p.group_m, m_blk, n_blk);
        const int a_row = m_blk * C::TILE_M + (int)rank * 128;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, ctl, 0, kWaitEmpty)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = sA + stage * C::A_BYTES;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          const int k0 = kb * BK;
          if constexpr (PAIR) {
            // Both CTAs' bytes complete on the leader's full barrier.
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if constexpr (!A_MN) {
              tma_load_2d_pair(a_dst, &tmA, bar, k0, a_row, hint_a);
            } else {
#pragma unroll
              for (int c = 0; c < 2; ++c) tma_load_2d_pair(a_dst + c * MN_CHUNK_BYTES, &tmA, bar, a_row + c * 64, k0, hint_a);
            }
            if constexpr (EPI == EPI_SWIGLU) {
              // Leader holds the 128 gate rows, the peer the 128 up rows of these output columns.
              tma_load_2d_pair(b_dst, &tmB, bar, k0, (rank ? p.split : 0) + n_blk * (BN / 2), hint_b);
            } else if constexpr (!B_MN) {
              tma_load_2d_pair(b_dst, &tmB, bar, k0, n_blk * BN + (int)rank * 128, hint_b);
            } else {
#pragma unroll
              for (int c = 0; c < 2; ++c)
                tma_load_2d_pair(b_dst + c * MN_CHUNK_BYTES, &tmB, bar, n_blk * BN + (int)rank * 128 + c * 64, k0, hint_b);
            }
          } else {
            uint64_t* bar = &full[stage];
            mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
            if constexpr (!A_MN) {
              tma_load_2d(a_dst, &tmA, bar, k0, a_row, hint_a);
            } else {
#pragma unroll
              for (int c = 0; c < 2; ++c) tma_load_2d(a_dst + c * MN_CHUNK_BYTES, &tmA, bar, a_row + c * 64, k0, hint_a);
            }
            if constexpr (EPI == EPI_SWIGLU) {
              tma_load_2d(b_dst, &tmB, bar, k0, n_blk * (BN / 2), hint_b);
              tma_load_2d(b_dst + C::B_BYTES / 2, &tmB, bar, k0, p.split + n_blk * (BN / 2), hint_b);
            } else if constexpr (!B_MN) {
              tma_load_2d(b_dst, &tmB, bar, k0, n_blk * BN, hint_b);
            } else {
#pragma unroll
              for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * MN_CHUNK_BYTES, &tmB, bar, n_blk * BN + c * 64, k0, hint_b);
            }
          }
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issuer (pair leader)
      constexpr uint32_t idesc = make_idesc_bf16(C::MMA_M, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = first_tile; tile < num_tiles && ok; tile += tile_step) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, ctl, 1, kWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, ctl, 1, kWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            // K-major: advance 16 elements (32 B) inside the 128-B swizzled row;
            // MN-major: advance 16 k-rows of 128 B (2 KiB), chunks of 64 mn 8 KiB apart.
            const uint64_t ad = A_MN ? make_sdesc_sw128(a_base + k * 2048, MN_CHUNK_BYTES, 1024)
                                     : make_sdesc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? make_sdesc_sw128(b_base + k * 2048, MN_CHUNK_BYTES, 1024)
                                     : make_sdesc_sw128(b_base + k * 32, 16, 1024);
            if constexpr (PAIR) umma_bf16_pair(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
            else umma_bf16(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          // Free the stage (in both CTAs of a pair) once these MMAs have read it.
          if constexpr (PAIR) {
            umma_commit_pair_both(&empty[stage]);
          } else {
            umma_commit(&empty[stage]);
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        // Accumulator ready for the epilogue warps (of both CTAs of a pair).
        if constexpr (PAIR) {
          umma_commit_pair_both(&tfull[acc]);
        } else {
          umma_commit(&tfull[acc]);
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Every MMA issued by this thread has completed once mma_done fires.
      if constexpr (PAIR) umma_commit_pair(mapa_shared(smem_u32(mma_done), 0));
      else umma_commit(mma_done);
      mbar_wait(mma_done, 0, ctl, 1, kWaitDrain);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (every CTA)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    EpiStore es;
    es.stg = sEpi + (warp - 2) * kEpiWarpBytes;
    es.lane = lane;
    es.rows = p.M;
    es.n = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = first_tile; tile < num_tiles; tile += tile_step) {
      int m_blk, n_blk;
      tile_coords(tile, p.num_m_tiles, p.num_n_tiles, p.group_m, m_blk, n_blk);
      const int row0 = m_blk * C::TILE_M + (int)rank * 128 + q * 32;
      Pref32 x0, x1;
      float rr = 1.f;
      epilogue_prefetch<EPI>(p, row0 + lane, row0 + lane < p.M, n_blk, x0, x1, rr);
      // Warp-uniform outcome: tcgen05.ld below needs all 32 lanes converged.
      const bool ok = mbar_wait(&tfull[acc], acc_phase, ctl, 2 + q, kWaitAccFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      es.row0 = row0;
      es.begin_tile();
      epilogue_tile<EPI>(p, tbase, row0 + lane, row0 + lane < p.M, row0 / 32, n_blk, lane, es, &tmO1, &tmO2, x0,
                         x1, rr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
        else mbar_arrive(&tempty[acc]);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    es.finish();  // every tile store has completed before the CTA's shared memory is released
  }

  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  if (*abort_flag) {
    // A role gave up: let the last (up to STAGES) copies land before shared
    // memory is released.  Every wait here is bounded too.
    if (warp == 0 && lane == 0 && rank == 0) {
      const int first = issued > S ? issued - S : 0;
      for (int i = first; i < issued; ++i) {
        const uint32_t par = (uint32_t)((i / S) & 1);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full[i % S], par) && global_timer_ns() - t0 < ctl.limit_ns) {
        }
      }
    }
    __syncthreads();
  }
  if constexpr (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace coda
