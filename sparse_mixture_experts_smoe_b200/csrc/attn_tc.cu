// attn_tc.cu -- the Mixture-of-Attention core on the 5th-generation tensor cores.
//
// What the pages ask for: ParallelLinear extended to Mixture of Attention (arXiv
// abstract), implemented without additional memory costs (tradepoint.io article,
// method paragraph).  The reading here: per-expert query projections produce, for
// slot p = t*kslots + j, a query row in grouped order (row inv[p] of q); keys and
// values are shared by the experts, [T, heads*128] in token order; the T tokens
// form sequences of L consecutive tokens; every head attends causally within its
// sequence:
//   o[inv[p], head] = softmax_u( <q, k_u> / sqrt(128) ) v_u,  u in [seq start, t]
// and o stays in grouped order for the per-expert output projection.  No grouped
// copy of anything is made: the query (and dO) rows of a tile are gathered through
// inv straight into shared memory.
//
// A query tile is 128 rows: tpt = 128 / kslots consecutive tokens, each with its
// kslots slots (the kslots queries of a token see the same keys).  Key blocks are
// 128 tokens.  Each kernel is warp-specialised: warp 0 issues TMA loads of key and
// value blocks, warp 1 issues tcgen05.mma (accumulators in tensor memory), warps
// 4-7 own one accumulator lane each (one query row, or one key row in the dK/dV
// kernel) and run the softmax arithmetic between the MMAs, writing the bf16
// probabilities (or score gradients) back into tensor memory, where the next MMA
// reads its A operand.
//
//   forward  : S = Q K^T -> online softmax (base 2, lazy rescale of O) -> O += P V;
//              o = O / l (bf16, grouped rows), lse = m + log l (fp32).  96 KB of
//              shared memory and 256 tensor-memory columns, so two CTAs share an SM
//              and one's softmax overlaps the other's MMAs.
//   backward : D = <dO, O> per row; dQ per query tile over its key blocks
//              (S, dP = dO V^T -> dS = P (dP - D) -> dQ += dS K); dK, dV per key
//              block over the query tiles that see it (S^T = K Q^T, dP^T = V dO^T
//              -> P^T, dS^T -> dV += P^T dO, dK += dS^T Q).  No atomics: each output
//              row is written once, so results are run-to-run identical.
//
// Every mbarrier wait is bounded (2 s); on expiry the kernel records the timeout,
// stops issuing work and frees its tensor memory.
#include "tc_ptx.cuh"

namespace smoe {
namespace {

constexpr int kDh = 128;                 // head width of these kernels
constexpr int kRows = 128;               // query rows per tile = keys per block (MMA M, N)
constexpr int kHalf = kRows * 64 * 2;    // one 64-column half of a 128 x 128 bf16 tile (16 KB)
constexpr int kTile = 2 * kHalf;         // 32 KB
constexpr int kAttnThreads = 256;        // 8 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLazy = 8.0f;            // rescale O only when the row max grows by > 2^8

struct AttnArgs {
  const bf16* q;        // [S, heads*128] grouped
  const bf16* k;        // [T, heads*128]
  const bf16* v;        // [T, heads*128]
  const bf16* dout;     // [S, heads*128] grouped (backward)
  const float* lse;     // [S, heads] (backward input)
  const float* dsum;    // [S, heads] = <dO, O> (backward)
  bf16* o;              // forward output
  float* lse_out;       // forward output
  bf16* dq;             // backward outputs
  bf16* dk;
  bf16* dv;
  const int32_t* inv;   // [S] grouped row of each slot
  int T, L, kslots, heads;
  int tpt;              // tokens per query tile
  int tiles_per_seq;    // query tiles per sequence
  int kv_per_seq;       // key blocks per sequence
  int nseq;
  unsigned* err;
};

// Query tile geometry: tokens [tb, te) of sequence s (starting at s0, ending at s1).
struct QTile {
  int s0, s1, tb, te;
  __device__ __forceinline__ void init(const AttnArgs& a, int s, int qt) {
    s0 = s * a.L;
    s1 = min(a.T, s0 + a.L);
    tb = s0 + qt * a.tpt;
    te = min(s1, tb + a.tpt);
  }
  // grouped row of tile row r, or -1 (padding, or an inverse entry out of range,
  // which a sorted_slot that is not a permutation leaves behind: reported); its
  // token in *t
  __device__ __forceinline__ int row(const AttnArgs& a, int r, int* t) const {
    const int tt = tb + r / a.kslots;
    *t = tt;
    if (r >= a.tpt * a.kslots || tt >= te) return -1;
    const int g = a.inv[(size_t)tt * a.kslots + r % a.kslots];
    if (g < 0 || g >= a.T * a.kslots) {
      report_error(a.err, ERRBIT_DATA);
      return -1;
    }
    return g;
  }
};

// One 128-byte swizzled 128 x 128 tile row (256 bytes = 16 chunks) gathered by
// cp.async: the two 64-column halves are 16 KB apart.  A missing row (src null) is
// zero-filled; its copies read nothing but still name a valid address (any).
__device__ __forceinline__ void gather_tile_row(uint32_t tile, const bf16* src, const bf16* any, int r) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t dst = tile + (c >> 3) * kHalf + sw128_off(r, c & 7);
    cp_async16(dst, src ? src + 8 * c : any, src ? 16u : 0u);
  }
}

// Descriptors of a 128 x 128 tile (two 64-column halves of 128 rows):
//   K-major (rows = M or N, 128 columns = the reduction): K-step kk of 16 columns;
//   MN-major (rows = the reduction, columns = N): K-step kk of 16 rows, the two
//   64-column halves 16 KB apart.
__device__ __forceinline__ uint64_t tile_kmajor(uint32_t base, int kk) {
  return desc_kmajor(base + (kk >> 2) * kHalf + (kk & 3) * 32);
}
__device__ __forceinline__ uint64_t tile_mnmajor(uint32_t base, int kk) {
  return sw128_desc(base + kk * 2048, kHalf, 1024);
}
constexpr uint32_t kIdescKK = idesc_bf16(kRows, kRows, 0, 0);  // A K-major, B K-major
constexpr uint32_t kIdescKM = idesc_bf16(kRows, kDh, 0, 1);    // A K-major (tensor memory), B MN-major

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// 32 values of a row as 16 packed bf16 pairs into tensor-memory columns [col, col + 16)
__device__ __forceinline__ void tmem_st_bf16x32(uint32_t taddr, const float* v) {
  uint32_t r[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) r[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
  tmem_st16(taddr, r);
}

struct AttnCtl {
  uint64_t bar[16];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void attn_setup(AttnCtl& c, const uint32_t* counts, int nbar, uint32_t cols) {
  if (threadIdx.x == 0) {
    for (int b = 0; b < nbar; ++b) mbar_init(&c.bar[b], counts[b]);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if ((threadIdx.x >> 5) == 1) tmem_alloc(&c.tmem_base, cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}
__device__ __forceinline__ void attn_teardown(AttnCtl& c, uint32_t cols) {
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  if (*reinterpret_cast<volatile int*>(&c.abort_flag)) {
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 2000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 1) tmem_dealloc(c.tmem_base, cols);
}

// Work item w -> (head, sequence, query tile), longest tiles (latest in their
// sequence) first so that the causal imbalance does not leave a tail.
__device__ __forceinline__ void qtile_of(const AttnArgs& a, int w, int& head, int& s, int& qt) {
  head = w % a.heads;
  const int lin = w / a.heads;
  s = lin % a.nseq;
  qt = a.tiles_per_seq - 1 - lin / a.nseq;
}

// ---------------------------------------------------------------------------
// Forward
// ---------------------------------------------------------------------------
// Barriers: 0 qfull (128 gather threads), 1 kfull, 2 kempty, 3 vfull, 4 vempty,
// 5 sfull, 6 pfull (4 softmax warps), 7 pvdone.
__global__ void __launch_bounds__(kAttnThreads, 2)
moa_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTile;
  uint8_t* sV = smem + 2 * kTile;
  AttnCtl& c = *reinterpret_cast<AttnCtl*>(smem + 3 * kTile);
  volatile int* abort_flag = &c.abort_flag;
  enum { QFULL, KFULL, KEMPTY, VFULL, VEMPTY, SFULL, PFULL, PVDONE, NBAR };
  const uint32_t counts[NBAR] = {128, 1, 1, 1, 1, 1, 4, 1};
  attn_setup(c, counts, NBAR, 256);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int head, s, qt;
  qtile_of(a, blockIdx.x, head, s, qt);
  QTile tl;
  tl.init(a, s, qt);
  const int nkv = tl.te > tl.tb ? cdiv(tl.te - tl.s0, kRows) : 0;
  const int W = a.heads * kDh;
  const uint32_t tS = c.tmem_base, tO = c.tmem_base + 128;

  if (warp == 0) {
    // ---------------- TMA producer: key and value blocks ----------------
    if (lane == 0) {
      for (int j = 0; j < nkv; ++j) {
        const uint32_t ph = j & 1;
        const int row0 = tl.s0 + j * kRows;
        if (!mbar_wait(&c.bar[KEMPTY], ph ^ 1, abort_flag, a.err)) break;
        mbar_expect_tx(&c.bar[KFULL], kTile);
        tma_load_2d(sK, &tmK, &c.bar[KFULL], head * kDh, row0);
        tma_load_2d(sK + kHalf, &tmK, &c.bar[KFULL], head * kDh + 64, row0);
        if (!mbar_wait(&c.bar[VEMPTY], ph ^ 1, abort_flag, a.err)) break;
        mbar_expect_tx(&c.bar[VFULL], kTile);
        tma_load_2d(sV, &tmV, &c.bar[VFULL], head * kDh, row0);
        tma_load_2d(sV + kHalf, &tmV, &c.bar[VFULL], head * kDh + 64, row0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && nkv > 0) {
      const uint32_t q_s = smem_u32(sQ), k_s = smem_u32(sK), v_s = smem_u32(sV);
      for (int j = 0; j < nkv; ++j) {
        const uint32_t ph = j & 1;
        if (j == 0 && !mbar_wait(&c.bar[QFULL], 0, abort_flag, a.err)) break;
        if (!mbar_wait(&c.bar[KFULL], ph, abort_flag, a.err)) break;
        // S and the previous block's P share columns: P V of block j-1 must be done
        if (j > 0 && !mbar_wait(&c.bar[PVDONE], ph ^ 1, abort_flag, a.err)) break;
        tc_fence_after();
        if (j == 0) fence_proxy_async();  // gathered query rows -> tensor core
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          umma_bf16(tS, tile_kmajor(q_s, kk), tile_kmajor(k_s, kk), kIdescKK, kk > 0);
        umma_commit(&c.bar[SFULL]);
        umma_commit(&c.bar[KEMPTY]);
        if (!mbar_wait(&c.bar[PFULL], ph, abort_flag, a.err)) break;
        if (!mbar_wait(&c.bar[VFULL], ph, abort_flag, a.err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          umma_bf16_ts(tO, tS + 8 * kk, tile_mnmajor(v_s, kk), kIdescKM, (j | kk) != 0);
        umma_commit(&c.bar[PVDONE]);
        umma_commit(&c.bar[VEMPTY]);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- query gather, softmax, output ----------------
    const int q4 = warp - 4;
    const int r = q4 * 32 + lane;
    int t_r;
    const int grow = tl.row(a, r, &t_r);
    gather_tile_row(smem_u32(sQ), grow >= 0 ? a.q + (size_t)grow * W + head * kDh : nullptr, a.q, r);
    cp_async_arrive(&c.bar[QFULL]);
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sc = kLog2e * rsqrtf((float)kDh);  // scores -> base-2 exponent
    float m_ref = 0.0f, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv && ok; ++j) {
      const uint32_t ph = j & 1;
      if (!mbar_wait(&c.bar[SFULL], ph, abort_flag, a.err)) { ok = false; break; }
      tc_fence_after();
      const int u0 = tl.s0 + j * kRows;
      // pass 1: the block's row maximum (masked keys: u > t, or past the sequence)
      float mb = -INFINITY;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(tS + lane_off + 32 * cc, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int u = u0 + 32 * cc + i;
          const bool keep = grow < 0 || (u <= t_r);
          if (keep) mb = fmaxf(mb, v[i] * sc);
        }
      }
      // reference maximum: the first block's, raised only when a row's maximum
      // grows by more than 2^kLazy (then O and l are rescaled); a warp rescales
      // together because tensor-memory loads and stores are warp-collective
      float m_new = m_ref;
      bool resc = false;
      if (j == 0) {
        m_new = mb;
      } else if (mb > m_ref + kLazy) {
        m_new = mb;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc)) {
        const float f = resc ? ex2(m_ref - m_new) : 1.0f;
        l *= f;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float v[32];
          tmem_ld32(tO + lane_off + 32 * cc, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= f;
          tmem_st32f(tO + lane_off + 32 * cc, v);
        }
      }
      m_ref = m_new;
      // pass 2: probabilities in bf16 over the score columns (chunk cc's 32 values
      // land in columns [16 cc, 16 cc + 16), which hold scores already consumed)
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(tS + lane_off + 32 * cc, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int u = u0 + 32 * cc + i;
          const bool keep = grow < 0 || (u <= t_r);
          const float p = keep ? ex2(v[i] * sc - m_ref) : 0.0f;
          l += p;
          v[i] = p;
        }
        tmem_st_bf16x32(tS + lane_off + 16 * cc, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.bar[PFULL]);
    }
    // output: O / l for this row, after the last P V
    if (ok && nkv > 0 && mbar_wait(&c.bar[PVDONE], (nkv - 1) & 1, abort_flag, a.err)) {
      tc_fence_after();
      const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
      bf16* dst = grow >= 0 ? a.o + (size_t)grow * W + head * kDh : nullptr;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(tO + lane_off + 32 * cc, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= inv_l;
        if (dst) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            *reinterpret_cast<uint4*>(dst + 32 * cc + 8 * h) = pack8(v + 8 * h);
        }
      }
      if (grow >= 0) a.lse_out[(size_t)grow * a.heads + head] = (m_ref + __log2f(l)) * kLn2;
    }
  }
  attn_teardown(c, 256);
}

// ---------------------------------------------------------------------------
// Backward, step 1: D = <dO, O> per (grouped row, head), fp32.  One warp per row.
// ---------------------------------------------------------------------------
__global__ void attn_dsum_kernel(const bf16* __restrict__ dout, const bf16* __restrict__ o, int S,
                                 int heads, float* __restrict__ dsum) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= S) return;
  const int W = heads * kDh;
  for (int h = 0; h < heads; ++h) {
    const uint2 a = *reinterpret_cast<const uint2*>(dout + (size_t)row * W + h * kDh + 4 * lane);
    const uint2 b = *reinterpret_cast<const uint2*>(o + (size_t)row * W + h * kDh + 4 * lane);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float2 fa = __bfloat1622float2(pa[i]), fb = __bfloat1622float2(pb[i]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dsum[(size_t)row * heads + h] = acc;
  }
}

// ---------------------------------------------------------------------------
// Backward, step 2: dQ per query tile.
// Barriers: 0 qfull (128), 1-2 kvfull[2], 3-4 kvempty[2], 5 sfull, 6 pfull (4), 7 tdone.
// Tensor memory: S [0,128) (dS written over it), dP [128,256), dQ [256,384).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kAttnThreads, 1)
moa_attn_dq_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sO = smem + kTile;                 // dO tile
  uint8_t* sKV = smem + 2 * kTile;            // 2 stages of (K, V)
  AttnCtl& c = *reinterpret_cast<AttnCtl*>(smem + 6 * kTile);
  volatile int* abort_flag = &c.abort_flag;
  enum { QFULL, KVFULL0, KVFULL1, KVEMPTY0, KVEMPTY1, SFULL, PFULL, TDONE, NBAR };
  const uint32_t counts[NBAR] = {128, 1, 1, 1, 1, 1, 4, 1};
  attn_setup(c, counts, NBAR, 512);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int head, s, qt;
  qtile_of(a, blockIdx.x, head, s, qt);
  QTile tl;
  tl.init(a, s, qt);
  const int nkv = tl.te > tl.tb ? cdiv(tl.te - tl.s0, kRows) : 0;
  const int W = a.heads * kDh;
  const uint32_t tS = c.tmem_base, tP = c.tmem_base + 128, tQ = c.tmem_base + 256;

  if (warp == 0) {
    if (lane == 0) {
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int row0 = tl.s0 + j * kRows;
        if (!mbar_wait(&c.bar[KVEMPTY0 + st], ph ^ 1, abort_flag, a.err)) break;
        uint8_t* kd = sKV + st * 2 * kTile;
        mbar_expect_tx(&c.bar[KVFULL0 + st], 2 * kTile);
        tma_load_2d(kd, &tmK, &c.bar[KVFULL0 + st], head * kDh, row0);
        tma_load_2d(kd + kHalf, &tmK, &c.bar[KVFULL0 + st], head * kDh + 64, row0);
        tma_load_2d(kd + kTile, &tmV, &c.bar[KVFULL0 + st], head * kDh, row0);
        tma_load_2d(kd + kTile + kHalf, &tmV, &c.bar[KVFULL0 + st], head * kDh + 64, row0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && nkv > 0) {
      const uint32_t q_s = smem_u32(sQ), o_s = smem_u32(sO);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const uint32_t k_s = smem_u32(sKV + st * 2 * kTile), v_s = k_s + kTile;
        if (j == 0 && !mbar_wait(&c.bar[QFULL], 0, abort_flag, a.err)) break;
        if (!mbar_wait(&c.bar[KVFULL0 + st], ph, abort_flag, a.err)) break;
        if (j > 0 && !mbar_wait(&c.bar[TDONE], (j - 1) & 1, abort_flag, a.err)) break;
        tc_fence_after();
        if (j == 0) fence_proxy_async();
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          umma_bf16(tS, tile_kmajor(q_s, kk), tile_kmajor(k_s, kk), kIdescKK, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          umma_bf16(tP, tile_kmajor(o_s, kk), tile_kmajor(v_s, kk), kIdescKK, kk > 0);
        umma_commit(&c.bar[SFULL]);
        if (!mbar_wait(&c.bar[PFULL], j & 1, abort_flag, a.err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          umma_bf16_ts(tQ, tS + 8 * kk, tile_mnmajor(k_s, kk), kIdescKM, (j | kk) != 0);
        umma_commit(&c.bar[TDONE]);
        umma_commit(&c.bar[KVEMPTY0 + st]);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int q4 = warp - 4;
    const int r = q4 * 32 + lane;
    int t_r;
    const int grow = tl.row(a, r, &t_r);
    gather_tile_row(smem_u32(sQ), grow >= 0 ? a.q + (size_t)grow * W + head * kDh : nullptr, a.q, r);
    gather_tile_row(smem_u32(sO), grow >= 0 ? a.dout + (size_t)grow * W + head * kDh : nullptr, a.dout, r);
    cp_async_arrive(&c.bar[QFULL]);
    const float lse2 = grow >= 0 ? a.lse[(size_t)grow * a.heads + head] * kLog2e : 0.0f;
    const float Dr = grow >= 0 ? a.dsum[(size_t)grow * a.heads + head] : 0.0f;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sc = kLog2e * rsqrtf((float)kDh);
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&c.bar[SFULL], j & 1, abort_flag, a.err)) { ok = false; break; }
      tc_fence_after();
      const int u0 = tl.s0 + j * kRows;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float sv[32], dp[32];
        tmem_ld32(tS + lane_off + 32 * cc, sv);
        tmem_ld32(tP + lane_off + 32 * cc, dp);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int u = u0 + 32 * cc + i;
          const bool keep = grow >= 0 && u <= t_r;
          const float p = keep ? ex2(sv[i] * sc - lse2) : 0.0f;
          sv[i] = p * (dp[i] - Dr);
        }
        tmem_st_bf16x32(tS + lane_off + 16 * cc, sv);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.bar[PFULL]);
    }
    if (ok && nkv > 0 && mbar_wait(&c.bar[TDONE], (nkv - 1) & 1, abort_flag, a.err)) {
      tc_fence_after();
      const float scale = rsqrtf((float)kDh);
      bf16* dst = grow >= 0 ? a.dq + (size_t)grow * W + head * kDh : nullptr;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(tQ + lane_off + 32 * cc, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= scale;
        if (dst) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            *reinterpret_cast<uint4*>(dst + 32 * cc + 8 * h) = pack8(v + 8 * h);
        }
      }
    }
  }
  attn_teardown(c, 512);
}

// ---------------------------------------------------------------------------
// Backward, step 3: dK and dV per key block of 128 keys, over the query tiles of
// its sequence that see it.  Warps 2-3 gather the query and dO rows of each tile
// (two stages) with the rows' lse (base 2), D and token; warps 4-7 own one key row.
// Barriers: 0 kvfull, 1-2 qfull[2] (64 cp.async + 64 stats arrivals), 3-4 qempty[2],
// 5 sfull, 6 pfull (4), 7 tdone.
// Tensor memory: S^T [0,128) (P^T over it), dP^T [128,256) (dS^T over it),
// dV [256,384), dK [384,512).
// ---------------------------------------------------------------------------
struct TileStats {
  float lse2[kRows];
  float D[kRows];
  int tok[kRows];  // token of the query row, -1 for padding
};

__global__ void __launch_bounds__(kAttnThreads, 1)
moa_attn_dkv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sK = smem;
  uint8_t* sV = smem + kTile;
  uint8_t* sQO = smem + 2 * kTile;  // stage st: Q at st * 2 kTile, dO after it
  TileStats* stats = reinterpret_cast<TileStats*>(smem + 6 * kTile);
  AttnCtl& c = *reinterpret_cast<AttnCtl*>(smem + 6 * kTile + 2 * sizeof(TileStats));
  volatile int* abort_flag = &c.abort_flag;
  enum { KVFULL, QFULL0, QFULL1, QEMPTY0, QEMPTY1, SFULL, PFULL, TDONE, NBAR };
  const uint32_t counts[NBAR] = {1, 128, 128, 1, 1, 1, 4, 1};
  attn_setup(c, counts, NBAR, 512);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work item -> (head, sequence, key block); latest key blocks last (they see the
  // fewest query tiles), so the heaviest start first
  const int head = blockIdx.x % a.heads;
  const int lin = blockIdx.x / a.heads;
  const int s = lin % a.nseq;
  const int kb = lin / a.nseq;
  const int s0 = s * a.L, s1 = min(a.T, s0 + a.L);
  const int u0 = s0 + kb * kRows;  // first key of the block
  // query tiles of this sequence whose tokens reach u0: from the tile holding u0
  const int qt0 = (u0 - s0) / a.tpt;
  const int nq = u0 < s1 ? a.tiles_per_seq - qt0 : 0;
  const int W = a.heads * kDh;
  const uint32_t tS = c.tmem_base, tP = c.tmem_base + 128, tV = c.tmem_base + 256,
                 tK = c.tmem_base + 384;

  if (warp == 0) {
    if (lane == 0 && nq > 0) {
      mbar_expect_tx(&c.bar[KVFULL], 2 * kTile);
      tma_load_2d(sK, &tmK, &c.bar[KVFULL], head * kDh, u0);
      tma_load_2d(sK + kHalf, &tmK, &c.bar[KVFULL], head * kDh + 64, u0);
      tma_load_2d(sV, &tmV, &c.bar[KVFULL], head * kDh, u0);
      tma_load_2d(sV + kHalf, &tmV, &c.bar[KVFULL], head * kDh + 64, u0);
    }
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    // ---------------- query / dO gather with the rows' statistics ----------------
    const int g = threadIdx.x - 64;  // 0..63: rows g and g + 64 of each tile
    for (int i = 0; i < nq; ++i) {
      const int st = i & 1;
      const uint32_t ph = (i >> 1) & 1;
      if (!mbar_wait(&c.bar[QEMPTY0 + st], ph ^ 1, abort_flag, a.err)) break;
      QTile tl;
      tl.init(a, s, qt0 + i);
      const uint32_t q_s = smem_u32(sQO + st * 2 * kTile), o_s = q_s + kTile;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = g + 64 * h;
        int t;
        const int grow = tl.row(a, r, &t);
        gather_tile_row(q_s, grow >= 0 ? a.q + (size_t)grow * W + head * kDh : nullptr, a.q, r);
        gather_tile_row(o_s, grow >= 0 ? a.dout + (size_t)grow * W + head * kDh : nullptr, a.dout, r);
        stats[st].lse2[r] = grow >= 0 ? a.lse[(size_t)grow * a.heads + head] * kLog2e : 0.0f;
        stats[st].D[r] = grow >= 0 ? a.dsum[(size_t)grow * a.heads + head] : 0.0f;
        stats[st].tok[r] = grow >= 0 ? t : -1;
      }
      mbar_arrive(&c.bar[QFULL0 + st]);      // the statistics (release)
      cp_async_arrive(&c.bar[QFULL0 + st]);  // the rows, once they land
    }
  } else if (warp == 1) {
    if (lane == 0 && nq > 0) {
      const uint32_t k_s = smem_u32(sK), v_s = smem_u32(sV);
      if (mbar_wait(&c.bar[KVFULL], 0, abort_flag, a.err)) {
        for (int i = 0; i < nq; ++i) {
          const int st = i & 1;
          const uint32_t ph = (i >> 1) & 1;
          const uint32_t q_s = smem_u32(sQO + st * 2 * kTile), o_s = q_s + kTile;
          if (!mbar_wait(&c.bar[QFULL0 + st], ph, abort_flag, a.err)) break;
          if (i > 0 && !mbar_wait(&c.bar[TDONE], (i - 1) & 1, abort_flag, a.err)) break;
          tc_fence_after();
          fence_proxy_async();  // gathered rows -> tensor core
#pragma unroll
          for (int kk = 0; kk < kDh / 16; ++kk)
            umma_bf16(tS, tile_kmajor(k_s, kk), tile_kmajor(q_s, kk), kIdescKK, kk > 0);
#pragma unroll
          for (int kk = 0; kk < kDh / 16; ++kk)
            umma_bf16(tP, tile_kmajor(v_s, kk), tile_kmajor(o_s, kk), kIdescKK, kk > 0);
          umma_commit(&c.bar[SFULL]);
          if (!mbar_wait(&c.bar[PFULL], i & 1, abort_flag, a.err)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            umma_bf16_ts(tV, tS + 8 * kk, tile_mnmajor(o_s, kk), kIdescKM, (i | kk) != 0);
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            umma_bf16_ts(tK, tP + 8 * kk, tile_mnmajor(q_s, kk), kIdescKM, (i | kk) != 0);
          umma_commit(&c.bar[TDONE]);
          umma_commit(&c.bar[QEMPTY0 + st]);
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- probabilities and score gradients, per key row ----------------
    const int q4 = warp - 4;
    const int r = q4 * 32 + lane;
    const int u = u0 + r;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sc = kLog2e * rsqrtf((float)kDh);
    bool ok = true;
    for (int i = 0; i < nq; ++i) {
      const int st = i & 1;
      if (!mbar_wait(&c.bar[SFULL], i & 1, abort_flag, a.err)) { ok = false; break; }
      tc_fence_after();
      const TileStats& ts = stats[st];
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float sv[32], dp[32];
        tmem_ld32(tS + lane_off + 32 * cc, sv);
        tmem_ld32(tP + lane_off + 32 * cc, dp);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int qr = 32 * cc + jj;
          const int t = ts.tok[qr];
          const bool keep = t >= 0 && u <= t;
          const float p = keep ? ex2(sv[jj] * sc - ts.lse2[qr]) : 0.0f;
          dp[jj] = p * (dp[jj] - ts.D[qr]);
          sv[jj] = p;
        }
        tmem_st_bf16x32(tS + lane_off + 16 * cc, sv);
        tmem_st_bf16x32(tP + lane_off + 16 * cc, dp);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.bar[PFULL]);
    }
    if (ok && nq > 0 && mbar_wait(&c.bar[TDONE], (nq - 1) & 1, abort_flag, a.err)) {
      tc_fence_after();
      const bool valid = u < s1;
      const float scale = rsqrtf((float)kDh);
#pragma unroll 1
      for (int w2 = 0; w2 < 2; ++w2) {
        bf16* dst = valid ? (w2 == 0 ? a.dv : a.dk) + (size_t)u * W + head * kDh : nullptr;
        const uint32_t tacc = w2 == 0 ? tV : tK;
        const float f = w2 == 0 ? 1.0f : scale;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float v[32];
          tmem_ld32(tacc + lane_off + 32 * cc, v);
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) v[i2] *= f;
          if (dst) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
              *reinterpret_cast<uint4*>(dst + 32 * cc + 8 * h) = pack8(v + 8 * h);
          }
        }
      }
    }
  }
  attn_teardown(c, 512);
}

// 2-D map over [rows, cols] bf16 (row-major) with 64 x 128 boxes, 128-byte swizzle.
cudaError_t kv_map(CUtensorMap* m, const void* base, int rows, int cols) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)(rows > 0 ? rows : 1)};
  const uint64_t strides[1] = {(uint64_t)cols * 2};
  const uint32_t box[2] = {64, (uint32_t)kRows};
  return make_map(m, base, 2, dims, strides, box);
}

AttnArgs attn_args(int T, int L, int kslots, int heads, const int32_t* inv, unsigned* err) {
  AttnArgs a{};
  a.T = T;
  a.L = L;
  a.kslots = kslots;
  a.heads = heads;
  a.tpt = kRows / kslots;
  a.tiles_per_seq = cdiv(L, a.tpt);
  a.kv_per_seq = cdiv(L, kRows);
  a.nseq = cdiv(T, L);
  a.inv = inv;
  a.err = err;
  return a;
}

constexpr size_t kFwdSmem = 1024 + 3 * (size_t)kTile + sizeof(AttnCtl);
constexpr size_t kDqSmem = 1024 + 6 * (size_t)kTile + sizeof(AttnCtl);
constexpr size_t kDkvSmem = 1024 + 6 * (size_t)kTile + 2 * sizeof(TileStats) + sizeof(AttnCtl);
static_assert(2 * kFwdSmem <= 228 * 1024 - 2048, "two forward CTAs per SM");
static_assert(kDqSmem <= 232448 && kDkvSmem <= 232448, "shared memory");

}  // namespace

int attn_head_dim() { return kDh; }

cudaError_t launch_moa_attn_fwd(const void* q, const void* k, const void* v, const int32_t* inv, int T,
                                int L, int kslots, int heads, void* o, float* lse, unsigned* err,
                                cudaStream_t s) {
  CUtensorMap tk, tv;
  cudaError_t e = kv_map(&tk, k, T, heads * kDh);
  if (e != cudaSuccess) return e;
  if ((e = kv_map(&tv, v, T, heads * kDh)) != cudaSuccess) return e;
  AttnArgs a = attn_args(T, L, kslots, heads, inv, err);
  a.q = (const bf16*)q;
  a.o = (bf16*)o;
  a.lse_out = lse;
  if ((e = cudaFuncSetAttribute(moa_attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kFwdSmem)) != cudaSuccess)
    return e;
  const int grid = a.heads * a.nseq * a.tiles_per_seq;
  moa_attn_fwd_kernel<<<grid, kAttnThreads, kFwdSmem, s>>>(tk, tv, a);
  return cudaGetLastError();
}

// The backward's three launches (each is bracketed on its own by the caller).
struct AttnBwdPlan {
  CUtensorMap tk, tv;
  AttnArgs a;
};
static cudaError_t attn_bwd_plan(AttnBwdPlan& p, const void* q, const void* k, const void* v,
                                 const float* lse, const void* dout, const int32_t* inv, int T, int L,
                                 int kslots, int heads, void* dq, void* dk, void* dv, float* dsum,
                                 unsigned* err) {
  cudaError_t e = kv_map(&p.tk, k, T, heads * kDh);
  if (e != cudaSuccess) return e;
  if ((e = kv_map(&p.tv, v, T, heads * kDh)) != cudaSuccess) return e;
  p.a = attn_args(T, L, kslots, heads, inv, err);
  p.a.q = (const bf16*)q;
  p.a.dout = (const bf16*)dout;
  p.a.lse = lse;
  p.a.dsum = dsum;
  p.a.dq = (bf16*)dq;
  p.a.dk = (bf16*)dk;
  p.a.dv = (bf16*)dv;
  return cudaSuccess;
}

cudaError_t launch_attn_dsum(const void* dout, const void* o, int S, int heads, float* dsum, cudaStream_t s) {
  attn_dsum_kernel<<<cdiv(S, 8), 256, 0, s>>>((const bf16*)dout, (const bf16*)o, S, heads, dsum);
  return cudaGetLastError();
}

cudaError_t launch_attn_dq(const void* q, const void* k, const void* v, const float* lse,
                           const void* dout, const int32_t* inv, int T, int L, int kslots, int heads,
                           void* dq, const float* dsum, unsigned* err, cudaStream_t s) {
  AttnBwdPlan p;
  cudaError_t e = attn_bwd_plan(p, q, k, v, lse, dout, inv, T, L, kslots, heads, dq, nullptr, nullptr,
                                const_cast<float*>(dsum), err);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(moa_attn_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kDqSmem)) != cudaSuccess)
    return e;
  moa_attn_dq_kernel<<<p.a.heads * p.a.nseq * p.a.tiles_per_seq, kAttnThreads, kDqSmem, s>>>(p.tk, p.tv, p.a);
  return cudaGetLastError();
}

cudaError_t launch_attn_dkv(const void* q, const void* k, const void* v, const float* lse,
                            const void* dout, const int32_t* inv, int T, int L, int kslots, int heads,
                            void* dk, void* dv, const float* dsum, unsigned* err, cudaStream_t s) {
  AttnBwdPlan p;
  cudaError_t e = attn_bwd_plan(p, q, k, v, lse, dout, inv, T, L, kslots, heads, nullptr, dk, dv,
                                const_cast<float*>(dsum), err);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(moa_attn_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kDkvSmem)) != cudaSuccess)
    return e;
  moa_attn_dkv_kernel<<<p.a.heads * p.a.nseq * p.a.kv_per_seq, kAttnThreads, kDkvSmem, s>>>(p.tk, p.tv, p.a);
  return cudaGetLastError();
}

}  // namespace smoe
