// gemm_tc.cu -- bf16 grouped GEMMs of ParallelLinear on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory), fed by the tensor memory
// accelerator (TMA).
//
// What the pages ask for (tradepoint.io article, method paragraphs; library page
// of arXiv 2403.08245, review 2 summary): grouped matrix products over scattered
// groups, reading and writing token-ordered rows directly, with no grouped or
// padded copy of the input.  Here every tile belongs to one expert's contiguous
// slice of the expert-sorted slot list:
//   * grouped operands (rows already in expert order) arrive by 2-D/3-D TMA tiles;
//   * scattered operands (token rows) are gathered straight from the
//     token-ordered tensor by four producer warps with 16-byte cp.async copies
//     (eight threads per 128-byte row segment, written in the 128-byte swizzle
//     the tensor core reads; rows past the slice are zero-filled).  TMA gather4
//     was measured first and moved about 10 bytes per cycle per SM, too slow to
//     feed the tensor core; the load/store path sustains the 48 KB per 512-cycle
//     stage;
//   * weights arrive as 3-D TMA tiles of W[e] ([E, K, N]: MN-major operand) or of
//     W[e]^T (K-major operand) -- out-of-range rows/columns read as zero.
// Both operands are staged in 128-byte-swizzled shared memory and consumed by
// tcgen05.mma (kind::f16, bf16 in, fp32 accumulate) issued by one thread.
//
// Grouped-M kernel (forward, dx): persistent CTAs walk a tile list built from the
// expert offsets (expert-major; inside an expert, panels of M tiles walked M tile
// first, then N tile, so that the CTAs of one wave share input rows and weight
// columns in L2).  Warp roles: warp 0 = TMA producer,
// warp 1 = MMA issuer and tensor-memory owner, warps 4-7 = epilogue (thread r owns
// accumulator row r), warps 8-15 = row gather of a scattered operand (without a
// gather, warps 8-11 are a second epilogue group for the scaled store).  Two
// 256-column fp32 accumulators in tensor memory let the epilogue of one tile
// overlap the main loop of the next.  Epilogues: scaled store (gate), activation
// forward (H and A = gelu(H) or silu(Hg) * Hu), and the activation backward (gate
// gradient partial <dA', A>, g*A, dH = g dA' act'(H)); their bf16 rows in grouped
// order move through shared memory as 32 x 32 TMA boxes, scattered rows by
// per-row bulk copies.
//
// dW kernel: tile (e, m, n) of dW[e] = sum over the expert's rows r of
// A[r, m] * B[r, n]; the reduction runs over the slice rows, so both operands are
// MN-major 64-row slabs; rows past the slice end are zero-filled (gathered
// operand) or zeroed in shared memory before the last MMA of the tile.
//
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the kernel sets
// the timeout bit of the error word, stops issuing work and frees its tensor
// memory before returning.
#include "tc_ptx.cuh"

namespace smoe {
namespace {

constexpr int BM = 128;           // rows per tile (MMA M)
constexpr int BK = 64;            // K per stage: one 128-byte swizzle row of bf16
constexpr int BN = 256;           // MMA N
constexpr int kThreads = 512;        // 16 warps
constexpr int kGatherWarp0 = 8;       // first warp of the row gather
constexpr int kGatherThreads = 256;   // grouped-M kernel: warps 8-15 (or 8-11, below)
constexpr int kDwGatherThreads = 256; // dW kernel: warps 8-15 gather (more copies in flight)
constexpr int kDwThreads = 512;
// Warp roles.  Grouped-M kernel: 0 TMA, 1 MMA, 2-3 idle, 4-7 epilogue, 8-15 row
// gather (without a gather: 8-11 second epilogue group for EPI_STORE).  dW kernel: 0 TMA, 1 MMA, 2 source rows, 3 idle, 4-7 epilogue, 8-15
// row gather.  (Measured: a second epilogue warp set on 12-15 with a 4-warp
// gather was slower than this split.)  The role ranges must not overlap:
static_assert(kGatherWarp0 == 8 && kGatherWarp0 + kGatherThreads / 32 <= kThreads / 32,
              "grouped-M gather warps must fit the block");
static_assert(kGatherWarp0 + kDwGatherThreads / 32 <= kDwThreads / 32,
              "dW gather warps must fit the block");
constexpr uint32_t kTmemCols = 512;  // two BN-column fp32 accumulators
// Gathered products with K up to this (except SwiGLU's forward) use the short-K layout
// of the grouped kernel (4 gather warps, two epilogue groups, 3 stages); longer ones
// keep 8 gather warps.
constexpr int kShortK = 2048;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int kMaxE = 1024;

// Activation arithmetic of the bf16 epilogues: one sigmoid per element via the
// fast exponential and division, tanh from the hardware approximation.  Their
// relative errors (~1e-6 and ~5e-4) sit far below bf16 rounding (3.9e-3) of the
// stored results.
__device__ __forceinline__ float fast_sigmoid(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }
__device__ __forceinline__ float fast_tanh(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fast_gelu(float h) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * h, h * h, h);
  return 0.5f * h * (1.0f + fast_tanh(u));
}
__device__ __forceinline__ float fast_gelu_grad(float h) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * h, h * h, h);
  const float th = fast_tanh(u);
  const float du = 0.7978845608028654f * fmaf(3.0f * 0.044715f, h * h, 1.0f);
  return 0.5f * (1.0f + th) + 0.5f * h * (1.0f - th * th) * du;
}

// ---------------------------------------------------------------------------
// Shared state, stage rings and the tile list
// ---------------------------------------------------------------------------
// The grouped-M kernel keeps both operands of a stage in one ring (4 stages of
// 48 KB, 6 of 32 KB per CTA of a pair); the dW kernel keeps them in two rings of 4
// stages (16 KB A + 32 KB B) that advance together.  Either way the rings fill
// kRingBytes.
constexpr int kMaxStages = 8;
constexpr int IDX_STAGES = 8;            // slot-index ring of the dW gathers
constexpr int kRingBytes = 192 * 1024;

struct SharedCtl {
  uint64_t fullA[kMaxStages], emptyA[kMaxStages];  // emptyA frees a stage of both rings
  uint64_t fullB[kMaxStages];
  uint64_t tfull[2], tempty[2];
  uint64_t pfull[kMaxStages];   // pair leader: the other CTA's stage s has landed
  uint64_t ifull[IDX_STAGES];   // index ring: written by warp 2
  uint64_t iempty[IDX_STAGES];  // index ring: released by the 4 gather warps
  uint64_t ebar[8];             // per epilogue warp: its input boxes have landed
  uint32_t tmem_base;
  int abort_flag;
  int total_mtiles;
  int prefix[kMaxE + 1];  // M-tile prefix per expert
};

// Shared memory after SharedCtl, per kernel.
// dW kernel: the expert offsets and the slot-index ring.
struct DwExtra {
  int idx[IDX_STAGES][2][BK];  // source row per operand (A, B) of each stage row, -1 = zero
  float gsc[IDX_STAGES][BK];   // gate of each stage row (gated A rows only)
  int off[kMaxE + 1];          // expert offsets
  short order[kMaxE];          // experts by descending row count (ties: lower id)
};
// Grouped-M kernel: a staging area per epilogue warp for the output of one
// 32-column chunk of its 32 accumulator rows, used in one of two layouts:
//   boxed: three 2 KB boxes of 32 rows x 64 bytes in the 64-byte swizzle, each
//          written out by one TMA tensor store (the warp's rows are consecutive
//          rows of one expert's slice);
//   slots: per thread a 208-byte slot of up to three 64-byte row segments (or
//          one 128-byte fp32 one) written out by per-row bulk copies; the stride
//          of 13 x 16 bytes keeps 8 consecutive threads' 16-byte accesses on
//          distinct banks.
constexpr int kSlotBytes = 208;
constexpr int kBoxBytes = 32 * 64;
constexpr int kWarpStaging = 32 * kSlotBytes;  // 13 x 512: boxes stay 512-byte aligned
static_assert(3 * kBoxBytes <= kWarpStaging && kWarpStaging % 512 == 0, "staging layout");
constexpr int kStagingBytes = 4 * kWarpStaging;
// Launch flags of the grouped kernel: epilogue box stores / box loads, and B (an
// MN-major weight operand) through the slab view (one TMA load per run of
// 64-column slabs instead of one per slab).
enum : int { kBoxStores = 1, kBoxLoads = 2, kSlabB = 4 };

constexpr size_t kCtlBytes = (sizeof(SharedCtl) + 1023) / 1024 * 1024;
constexpr size_t kGroupedSmem = 1024 + (size_t)kRingBytes + kCtlBytes + kStagingBytes;
// dW kernel: after DwExtra, one 4 KB fp32 box (32 x 32, 128-byte swizzle) per
// epilogue warp, written out by a TMA tensor store per 32-column chunk.
constexpr size_t kDwExtraBytes = (sizeof(DwExtra) + 1023) / 1024 * 1024;
constexpr int kDwBoxBytes = 32 * 32 * 4;
constexpr size_t kDwSmem = 1024 + (size_t)kRingBytes + kCtlBytes + kDwExtraBytes + 4 * kDwBoxBytes;
static_assert(kGroupedSmem <= 232448 && kDwSmem <= 232448, "shared memory exceeds 227 KB");

// Position in a ring of n stages and the parity of the current lap.
struct Ring {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int n) {
    if (++s == n) { s = 0; ph ^= 1; }
  }
};

struct Tile {
  int e, mb, nb, row0, row_end;
};

// linear tile L -> (expert, M tile, N tile); expert-major, then panel, N tile, M tile.
// `off` = the expert offsets in global memory (validated by setup).
// A pair's M tile spans 2 BM rows, of which CTA `rank` takes the rank-th BM.
// Inside an expert the tiles go in panels of `pm` M tiles (the last panel may be
// shorter): M tile fastest, then N tile, then panel, so that the tiles in flight
// at once share fewer A rows (pm >= the expert's M tiles: one panel).
template <bool PAIR = false>
__device__ __forceinline__ Tile map_tile(const SharedCtl& c, const int32_t* off, int E, int nN,
                                         int L, int rank = 0, int pm = 1 << 30) {
  int lo = 0, hi = E - 1;  // largest e with prefix[e] * nN <= L
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (c.prefix[mid] * nN <= L) lo = mid; else hi = mid - 1;
  }
  Tile t;
  t.e = lo;
  const int mt = c.prefix[lo + 1] - c.prefix[lo];
  const int lp = L - c.prefix[lo] * nN;
  const int ph = pm < mt ? pm : mt;      // full panel height
  const int pan = lp / (ph * nN);        // panel index
  const int m0 = pan * ph;               // its first M tile
  const int h = min(ph, mt - m0);        // its height
  const int q = lp - pan * ph * nN;      // position inside the panel
  t.nb = q / h;
  t.mb = m0 + q % h;
  t.row0 = __ldg(off + lo) + t.mb * (PAIR ? 2 * BM : BM) + rank * BM;
  t.row_end = __ldg(off + lo + 1);
  return t;
}

// Setup common to both kernels: barriers, tensor memory, offsets (validated;
// copied to off_copy when given).
// a_arrivals / b_arrivals: producer arrivals per full stage (1 for TMA, the
// gather threads' cp.async arrivals otherwise).
template <int SA, int SB, bool PAIR = false>
__device__ __forceinline__ void setup(SharedCtl& c, const int32_t* offsets, int E, int num_rows,
                                      unsigned* err, uint32_t a_arrivals, uint32_t b_arrivals,
                                      uint32_t gather_warps, int* off_copy,
                                      uint32_t epilogue_warps = 4) {
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(&c.fullA[s], a_arrivals);
      mbar_init(&c.emptyA[s], 1);
      mbar_init(&c.pfull[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&c.fullB[s], b_arrivals);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c.tfull[b], 1);
      mbar_init(&c.tempty[b], epilogue_warps * (PAIR ? 2 : 1));  // a pair's leader: both CTAs' warps
    }
    for (int b = 0; b < IDX_STAGES; ++b) {
      mbar_init(&c.ifull[b], 1);
      mbar_init(&c.iempty[b], gather_warps);
    }
    for (int b = 0; b < 8; ++b) mbar_init(&c.ebar[b], 1);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if (PAIR) tmem_alloc_pair(&c.tmem_base, kTmemCols);
    else tmem_alloc(&c.tmem_base, kTmemCols);
  }
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {  // raw offsets first
    const int o = offsets[e];
    c.prefix[e] = o;
    if (off_copy) off_copy[e] = o;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // in place: offsets -> M-tile prefix
    bool ok = c.prefix[0] == 0 && c.prefix[E] == num_rows;
    int prev = c.prefix[0];
    c.prefix[0] = 0;
    for (int e = 0; e < E; ++e) {
      const int cur = c.prefix[e + 1];
      const int n = cur - prev;
      prev = cur;
      if (n < 0) ok = false;
      constexpr int TR = PAIR ? 2 * BM : BM;
      c.prefix[e + 1] = c.prefix[e] + (n > 0 ? (n + TR - 1) / TR : 0);
    }
    if (!ok) {  // inconsistent offsets: do nothing rather than read out of range
      report_error(err, ERRBIT_DATA);
      for (int e = 0; e <= E; ++e) c.prefix[e] = 0;
    }
    c.total_mtiles = c.prefix[E];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (PAIR) cluster_sync();  // both CTAs' barriers exist before either arrives remotely
}

// On an abort some copies (cp.async, TMA) and tensor-core operations may still
// be in flight: each thread retires its own cp.async copies, then the CTA waits
// a bounded 2 ms (far above any copy or MMA latency) before freeing tensor memory
// and exiting, so nothing lands in a CTA that has gone.
template <bool PAIR = false>
__device__ __forceinline__ void teardown(SharedCtl& c) {
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
  // a pair: neither CTA leaves while the other may still arrive on its barriers
  if (PAIR) cluster_sync();
  if ((threadIdx.x >> 5) == 1) {
    if (PAIR) tmem_dealloc_pair(c.tmem_base, kTmemCols);
    else tmem_dealloc(c.tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Grouped-M kernel
// ---------------------------------------------------------------------------
// F8: e4m3 operands (kind::f8f6f4, B K-major): a K-block is 128 values, i.e. the
// same 128 bytes per row as 64 bf16 values, so rings, swizzle and descriptors are
// unchanged; the epilogue multiplies the fp32 sums by the A row's scale and the
// weight column's scale before it does anything else.
template <bool A_GATHER, bool B_KMAJOR, bool SWIGLU_FWD, bool PAIR, bool SPLITK = false,
          bool SHORTK = false, bool F8 = false, bool G128 = false>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmO2,
                       const __grid_constant__ CUtensorMap tmXa,
                       const __grid_constant__ CUtensorMap tmXh, const GroupedGemm g, int nN,
                       int box_flags) {
  // One ring of STAGES stages holds A and B together (fullA/emptyA guard a whole
  // stage): measured faster here than separate rings, whose second wait and
  // commit per stage cost more than their extra depth returned.  A pair's CTA
  // holds half of B per stage, so its ring is deeper.  SHORTK (a gathered product
  // with a short K): 3 stages, half the gather warps (8-11), and warps 12-15 as a
  // second epilogue group staging in the ring space the fourth stage leaves free.
  // G128: a long-K gathered product with 4 gather warps (8-11) instead of 8: half
  // the per-stage barrier arrivals, measured faster on the tensor pipe.
  constexpr int BSTAGE = PAIR ? B_BYTES / 2 : B_BYTES;
  constexpr int STAGES = PAIR ? 6 : (SHORTK ? 3 : 4);
  constexpr int GTHREADS = (SHORTK || G128) ? 128 : kGatherThreads;  // gather threads
  static_assert(!G128 || (A_GATHER && !SHORTK), "4-warp gather of a long-K product");
  static_assert(!SHORTK || (A_GATHER && !PAIR &&
                            STAGES * (A_BYTES + BSTAGE) + 4 * kWarpStaging <= kRingBytes),
                "short-K layout");
  static_assert(STAGES * (A_BYTES + BSTAGE) <= kRingBytes, "stage ring exceeds its budget");
  static_assert(STAGES <= kMaxStages, "too many stages");
  static_assert(!F8 || (B_KMAJOR && !PAIR && !SHORTK), "FP8 products: K-major weights, one CTA");
  constexpr int BKE = F8 ? 2 * BK : BK;  // K values per stage (128 bytes per row either way)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  SharedCtl& c = *reinterpret_cast<SharedCtl*>(smem + kRingBytes);
  volatile int* abort_flag = &c.abort_flag;

  // a pair walks the tile list as one unit; rank 0 issues the MMAs.  Arrivals
  // on a stage's full barrier: the producer's expect-tx and the gather threads;
  // at a pair's rank 1 only its gather threads (relayed to the leader).
  const int rank = PAIR ? (int)cluster_rank() : 0;
  const uint32_t full_arrivals =
      (rank == 0 ? 1u : 0u) + (A_GATHER ? (uint32_t)GTHREADS : 0u);
  setup<STAGES, 0, PAIR>(c, g.offsets, g.E, g.num_rows, g.err, full_arrivals > 0 ? full_arrivals : 1u,
                         1, GTHREADS / 32, nullptr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int stride = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int nK = cdiv(g.K, BKE);
  // Split K (a product with too few tiles to fill the GPU, as at decode sizes):
  // work item L is K-blocks [kb_lo(L), kb_hi(L)) of tile L / ks, and the epilogue
  // stores the raw fp32 sum to its split's partial buffer (reduced afterwards).
  const int ks = SPLITK ? g.ksplit : 1;  // 1 (folded away) in every other instantiation
  const int total = c.total_mtiles * nN * ks;
  auto kb_lo = [&](int L) { return (L % ks) * nK / ks; };
  auto kb_hi = [&](int L) { return (L % ks + 1) * nK / ks; };
  constexpr int BNo = SWIGLU_FWD ? BN / 2 : BN;  // logical output columns per tile

  if (warp == 0) {
    // ---------------- TMA producer (weights; A too when grouped) ----------------
    if (lane == 0) {
      Ring r;
      bool run = true;
      for (int L = first; run && L < total; L += stride) {
        const Tile t = map_tile<PAIR>(c, g.offsets, g.E, nN, L / ks, rank, g.panel_m);
        for (int kb = kb_lo(L), kb_end = kb_hi(L); kb < kb_end; ++kb) {
          if (!mbar_wait(&c.emptyA[r.s], r.ph ^ 1, abort_flag, g.err)) { run = false; break; }
          uint8_t* b_dst = sB + r.s * BSTAGE;
          // a pair: both CTAs' TMA bytes count on the leader's barrier, whose
          // producer expects them all
          const uint32_t full_cl = PAIR ? peer_addr(&c.fullA[r.s], 0) : 0u;
          auto load2 = [&](void* dst, const CUtensorMap* m, int c0, int c1) {
            if (PAIR) tma_load_2d_pair(dst, m, full_cl, c0, c1);
            else tma_load_2d(dst, m, &c.fullA[r.s], c0, c1);
          };
          auto load3 = [&](void* dst, const CUtensorMap* m, int c0, int c1, int c2) {
            if (PAIR) tma_load_3d_pair(dst, m, full_cl, c0, c1, c2);
            else tma_load_3d(dst, m, &c.fullA[r.s], c0, c1, c2);
          };
          auto load4 = [&](void* dst, const CUtensorMap* m, int c0, int c1, int c2, int c3) {
            if (PAIR) tma_load_4d_pair(dst, m, full_cl, c0, c1, c2, c3);
            else tma_load_4d(dst, m, &c.fullA[r.s], c0, c1, c2, c3);
          };
          if (rank == 0)
            mbar_expect_tx(&c.fullA[r.s], (PAIR ? 2 : 1) * (BSTAGE + (A_GATHER ? 0 : A_BYTES)));
          if (!A_GATHER) load2(sA + r.s * A_BYTES, &tmA, kb * BKE, t.row0);
          if (B_KMAJOR && SWIGLU_FWD) {  // BNo gate rows, then BNo up rows of W[e]^T
            load3(b_dst, &tmB, kb * BKE, t.nb * BNo, t.e);
            load3(b_dst + BNo * 128, &tmB, kb * BKE, g.n_out + t.nb * BNo, t.e);
          } else if (B_KMAJOR) {  // rows of W[e] = output columns; a pair's CTA takes its half
            load3(b_dst, &tmB, kb * BKE, t.nb * BN + (PAIR ? rank * (BN / 2) : 0), t.e);
          } else if (box_flags & kSlabB) {
            // slab view: one load per contiguous column run (128 columns for SwiGLU's
            // gate and up halves and for a pair's half, else the tile's 256)
            constexpr int kRun = (PAIR || SWIGLU_FWD) ? BN / 2 : BN;
#pragma unroll
            for (int q = 0; q < BSTAGE / (kRun * BK * 2); ++q) {
              const int lc = (PAIR ? rank * (BN / 2) : 0) + kRun * q;  // column within the B tile
              const int col = SWIGLU_FWD ? (lc < BNo ? t.nb * BNo + lc : g.n_out + t.nb * BNo + lc - BNo)
                                         : t.nb * BN + lc;
              load4(b_dst + q * (kRun * BK * 2), &tmB, 0, kb * BK, col / 64, t.e);
            }
          } else {
            // 64-column slabs; SwiGLU's tile is BNo gate columns then BNo up columns
            // (a pair: the gate half in CTA 0, the up half in CTA 1)
#pragma unroll
            for (int q = 0; q < BSTAGE / (64 * BK * 2); ++q) {
              const int lc = (PAIR ? rank * (BN / 2) : 0) + 64 * q;  // column within the B tile
              const int col = SWIGLU_FWD ? (lc < BNo ? t.nb * BNo + lc : g.n_out + t.nb * BNo + lc - BNo)
                                         : t.nb * BN + lc;
              load3(b_dst + q * (64 * BK * 2), &tmB, col, kb * BK, t.e);
            }
          }
          r.next(STAGES);
        }
      }
    }
    __syncwarp();
  } else if (A_GATHER && warp >= kGatherWarp0 && warp < kGatherWarp0 + GTHREADS / 32) {
    // ---------------- row gather of the scattered A operand ----------------
    // thread t copies 16-byte chunk (t % 8) of tile rows t/8 + kRowStep j into
    // the 128-byte-swizzled K-major layout; rows past the expert's slice and
    // columns past K are zero-filled.
    // (addressed in bytes: a row is lda elements of 2 bytes, or of 1 for F8)
    constexpr int kRowStep = GTHREADS / 8, kRowsPer = BM / kRowStep;
    constexpr int ESZ = F8 ? 1 : 2;
    const int t = threadIdx.x - kGatherWarp0 * 32;
    const int cc = t & 7, r0 = t >> 3;
    const char* A = reinterpret_cast<const char*>(g.a);
    Ring r;
    bool run = true;
    for (int L = first; run && L < total; L += stride) {
      const Tile tl = map_tile<PAIR>(c, g.offsets, g.E, nN, L / ks, rank, g.panel_m);
      const char* src[kRowsPer];
      uint32_t ok_rows = 0;
#pragma unroll
      for (int j = 0; j < kRowsPer; ++j) {
        const int i = tl.row0 + r0 + kRowStep * j;
        src[j] = A;
        if (i < tl.row_end) {
          const int p = g.sorted_slot[i];
          const int xr = p / g.a_fan_out;
          if (p >= 0 && xr < g.a_rows) {
            src[j] = A + (size_t)xr * g.lda * ESZ + 16 * cc;
            ok_rows |= 1u << j;
          } else {
            report_error(g.err, ERRBIT_DATA);
          }
        }
      }
      for (int kb = kb_lo(L), kb_end = kb_hi(L); kb < kb_end; ++kb) {
        if (!mbar_wait(&c.emptyA[r.s], r.ph ^ 1, abort_flag, g.err)) { run = false; break; }
        const uint32_t a_dst = smem_u32(sA + r.s * A_BYTES);
        const bool col_ok = kb * 128 + 16 * cc < g.K * ESZ;
#pragma unroll
        for (int j = 0; j < kRowsPer; ++j) {
          const bool ok = col_ok && ((ok_rows >> j) & 1u);
          cp_async16(a_dst + sw128_off(r0 + kRowStep * j, cc), ok ? src[j] + kb * 128 : A, ok ? 16u : 0u);
        }
        cp_async_arrive(&c.fullA[r.s]);
        r.next(STAGES);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (a pair: rank 0; rank 1 relays its stages) ----------------
    if (lane == 0 && PAIR && rank == 1) {
      // the leader's MMAs read this CTA's half of each stage: its TMA bytes count
      // on the leader's barrier directly; its gathered rows are relayed from here
      if (A_GATHER) {
        Ring r;
        bool run = true;
        for (int L = first; run && L < total; L += stride) {
          for (int kb = kb_lo(L), kb_end = kb_hi(L); kb < kb_end; ++kb) {
            if (!mbar_wait(&c.fullA[r.s], r.ph, abort_flag, g.err)) { run = false; break; }
            fence_proxy_async();  // rows written by cp.async, read by the tensor core
            mbar_arrive_cluster_relaxed(peer_addr(&c.pfull[r.s], 0));
            r.next(STAGES);
          }
        }
      }
    } else if (lane == 0) {
      constexpr uint32_t idesc = F8 ? idesc_e4m3(BM, BN)
                                    : idesc_bf16(PAIR ? 2 * BM : BM, BN, 0, B_KMAJOR ? 0 : 1);
      Ring r;
      int it = 0;
      for (int L = first; L < total; L += stride, ++it) {
        const int buf = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!mbar_wait(&c.tempty[buf], tph ^ 1, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = c.tmem_base + buf * BN;
        const int kb0 = kb_lo(L);
        bool ok = true;
        for (int kb = kb_lo(L), kb_end = kb_hi(L); kb < kb_end; ++kb) {
          if (!mbar_wait(&c.fullA[r.s], r.ph, abort_flag, g.err)) { ok = false; break; }
          if (PAIR && A_GATHER && !mbar_wait(&c.pfull[r.s], r.ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          if (A_GATHER) fence_proxy_async();  // rows written by cp.async, read by the tensor core
          const uint32_t a_addr = smem_u32(sA + r.s * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + r.s * BSTAGE);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_kmajor(a_addr + kk * 32);
            const uint64_t bd = B_KMAJOR ? desc_kmajor(b_addr + kk * 32) : desc_mnmajor(b_addr + kk * 2048);
            if (PAIR) umma_bf16_pair(d_tmem, ad, bd, idesc, ((kb - kb0) | kk) != 0);
            else if (F8) umma_e4m3(d_tmem, ad, bd, idesc, ((kb - kb0) | kk) != 0);
            else umma_bf16(d_tmem, ad, bd, idesc, ((kb - kb0) | kk) != 0);
          }
          if (PAIR) {  // the stage is free in both CTAs
            umma_commit_pair_both(&c.emptyA[r.s]);
          } else {
            umma_commit(&c.emptyA[r.s]);
          }
          r.next(STAGES);
        }
        if (!ok) break;
        if (PAIR) {
          umma_commit_pair_both(&c.tfull[buf]);
        } else {
          umma_commit(&c.tfull[buf]);
        }
      }
    }
    __syncwarp();
  } else if ((warp >= 4 && warp < 8) ||
             (!A_GATHER && !SWIGLU_FWD && g.epi == EPI_STORE && warp >= 8 && warp < 12) ||
             (SHORTK && warp >= 12 && warp < 16)) {
    // warps 2-3 idle, and 8-15 without a gather except as below
    // ---------------- epilogue ----------------
    // Thread r owns accumulator row r.  Per 32-column chunk the warp stages its
    // rows' output segments in shared memory and hands them to the TMA engine:
    // one tensor store per output box when its 32 rows are consecutive rows of
    // the expert's slice (kBoxStores), else one bulk copy per row.  Plain stores
    // from the tensor-memory row layout would make every 16-byte access of a
    // warp touch 32 lines and compete with the cp.async row gathers for the same
    // unit.  ACT_BWD reads its A and H inputs the same way, as boxes of the
    // warp's rows (kBoxLoads), when they are in grouped order, else by 16-byte
    // loads issued before the accumulator read (per-row bulk loads of 64 bytes
    // measured far slower).
    // Without a gather, EPI_STORE runs two epilogue groups, warps 4-7 on the tiles
    // of accumulator buffer 0 and warps 8-11 on those of buffer 1, so that two
    // tiles drain at once (a short-K product's epilogue is longer than its MMAs).
    // A group stages in box `grp` of its quadrant's area; a warp whose rows leave
    // the slice stores them directly.
    // SHORTK: the same split of tiles by accumulator buffer for every epilogue, warps
    // 12-15 with staging areas of their own (so ragged rows use their slots).
    const bool shared_area = !A_GATHER && !SWIGLU_FWD && g.epi == EPI_STORE;
    const bool two = shared_area || SHORTK;
    const int grp = warp >= 8 ? 1 : 0;
    const int q = warp & 3;  // tensor-memory lane quadrant
    const int r = q * 32 + lane;
    uint8_t* wstage = (SHORTK && grp == 1)
                          ? smem + STAGES * (A_BYTES + BSTAGE) + q * kWarpStaging
                          : smem + kRingBytes + kCtlBytes + q * kWarpStaging;
    uint64_t* ebar = &c.ebar[grp * 4 + q];
    uint8_t* slot = wstage + lane * kSlotBytes;
    const uint32_t wstage_s = smem_u32(wstage), slot_s = smem_u32(slot);
    const int sw = (lane >> 1) & 3;  // 64-byte swizzle of this thread's box row
    const bf16* AUXA = reinterpret_cast<const bf16*>(g.aux_a);
    const bf16* AUXH = reinterpret_cast<const bf16*>(g.aux_h);
    // SwiGLU's forward instantiation has only the ACT_FWD epilogue
    const bool act_bwd = !SWIGLU_FWD && g.epi == EPI_ACT_BWD;
    const bool epi_store = !SWIGLU_FWD && g.epi == EPI_STORE;
    const bool swi = g.act == SMOE_ACT_SWIGLU;
    const bool need_h = act_bwd && g.out != nullptr && g.act != SMOE_ACT_NONE;
    uint32_t eph = 0;  // phase of this warp's input-box barrier
    int it = 0;
    for (int L = first; L < total; L += stride, ++it) {
      const int buf = it & 1;
      if (two && buf != grp) continue;  // the other group's tile
      const uint32_t tph = (it >> 1) & 1;
      const Tile t = map_tile<PAIR>(c, g.offsets, g.E, nN, L / ks, rank, g.panel_m);
      if (!mbar_wait(&c.tfull[buf], tph, abort_flag, g.err)) break;
      tc_fence_after();
      const int i = t.row0 + r;
      const bool valid = i < t.row_end;
      const int p = valid ? g.sorted_slot[i] : 0;
      const bool p_ok = valid && p >= 0 && p < g.num_rows;
      if (valid && !p_ok) report_error(g.err, ERRBIT_DATA);
      const int orow = g.out_mode == ROWS_GROUPED ? i : p;
      const float gate = (p_ok && g.gates) ? g.gates[p] : 1.0f;
      // F8: the scale of this row's A operand (its source row) and the weight
      // column scales of the tile's expert
      const float rs = (F8 && p_ok) ? (g.a_mode == ROWS_GATHER ? g.row_scale[p / g.a_fan_out] : g.row_scale[i])
                                    : 0.0f;
      const float* col_sc = F8 ? g.col_scale + (size_t)t.e * g.NW : nullptr;
      const uint32_t trow = c.tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
      const int wrow0 = t.row0 + q * 32;
      const bool boxed = (box_flags & kBoxStores) && wrow0 + 32 <= t.row_end;  // warp-uniform
      const bool direct = shared_area && !boxed;  // warp-uniform: plain stores from registers
      const int kb = shared_area ? grp : 0;       // first box of this warp's outputs
      // 16-byte chunk j8 of box k in this thread's row
      auto box_chunk = [&](int k, int j8) -> uint4* {
        return reinterpret_cast<uint4*>(wstage + k * kBoxBytes + lane * 64 + ((j8 ^ sw) << 4));
      };
      // 16-byte chunk j8 of output segment k of this thread's row
      auto chunk = [&](int k, int j8) -> uint4* {
        return reinterpret_cast<uint4*>(boxed ? wstage + (k + kb) * kBoxBytes + lane * 64 + ((j8 ^ sw) << 4)
                                              : slot + k * 64 + 16 * j8);
      };
      float dg_acc = 0.0f;
      int arow = 0;
      if (act_bwd && p_ok) arow = g.aux_a_mode == ROWS_GROUPED ? i : p / g.aux_a_fan_out;
#pragma unroll 1
      for (int c0 = 0; c0 < BNo; c0 += 32) {
        const int n0 = t.nb * BNo + c0;
        const int ncols = min(32, g.n_out - n0);  // a multiple of 8, uniform over the warp
        if (ncols <= 0) break;
        const uint32_t seg = (uint32_t)ncols * 2;  // bytes of the chunk's bf16 row segment
        float v[32], u[32];
        uint4 ra[4], rg[4], ru[4];
        if (act_bwd && (box_flags & kBoxLoads)) {
          // inputs as boxes of the warp's 32 rows (rows past the slice are read
          // but not used; rows past the tensor read as zeros)
          bulk_wait_read();
          __syncwarp();
          if (lane == 0) {
            const uint32_t nbox = 1u + (need_h ? 1u : 0u) + (need_h && swi ? 1u : 0u);
            mbar_expect_tx(ebar, nbox * kBoxBytes);
            tma_load_3d(wstage, &tmXa, ebar, n0, 0, wrow0);
            if (need_h) {
              tma_load_3d(wstage + kBoxBytes, &tmXh, ebar, n0, 0, wrow0);
              if (swi) tma_load_3d(wstage + 2 * kBoxBytes, &tmXh, ebar, n0, 1, wrow0);
            }
          }
          tmem_ld32(trow + c0, v);
          if (!mbar_wait(ebar, eph, abort_flag, g.err)) break;
          eph ^= 1;
#pragma unroll
          for (int j8 = 0; j8 < 4; ++j8) {
            ra[j8] = *box_chunk(0, j8);
            rg[j8] = need_h ? *box_chunk(1, j8) : make_uint4(0, 0, 0, 0);
            ru[j8] = (need_h && swi) ? *box_chunk(2, j8) : make_uint4(0, 0, 0, 0);
          }
          __syncwarp();  // every lane has read its rows before any lane writes
        } else if (act_bwd) {  // issue the chunk's global loads before the accumulator read
#pragma unroll
          for (int j8 = 0; j8 < 4; ++j8) {
            const int n = n0 + 8 * j8;
            const bool in = p_ok && 8 * j8 < ncols;
            const uint4 z = make_uint4(0, 0, 0, 0);
            ra[j8] = in ? __ldg(reinterpret_cast<const uint4*>(AUXA + (size_t)arow * g.ld_aux_a + n)) : z;
            rg[j8] = (in && need_h) ? __ldg(reinterpret_cast<const uint4*>(AUXH + (size_t)i * g.ld_aux_h + n)) : z;
            ru[j8] = (in && need_h && swi)
                         ? __ldg(reinterpret_cast<const uint4*>(AUXH + (size_t)i * g.ld_aux_h + g.n_out + n))
                         : z;
          }
        }
        if (!(act_bwd && (box_flags & kBoxLoads))) tmem_ld32(trow + c0, v);
        if (F8) {  // fp32 sum x (A row's scale) x (weight column's scale)
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 cs = 4 * q4 < ncols ? __ldg(reinterpret_cast<const float4*>(col_sc + n0 + 4 * q4))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * q4] *= rs * cs.x; v[4 * q4 + 1] *= rs * cs.y;
            v[4 * q4 + 2] *= rs * cs.z; v[4 * q4 + 3] *= rs * cs.w;
          }
        }
        if (SPLITK) {  // split K: this split's raw fp32 sums
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(
                g.partial + ((size_t)(L % ks) * g.num_rows + i) * g.n_out + n0);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              if (4 * q4 < ncols)
                dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
          }
          continue;
        }
        if (SWIGLU_FWD) tmem_ld32(trow + BNo + c0, u);
        if (F8 && SWIGLU_FWD) {  // the up half's columns start at n_out
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 cs = 4 * q4 < ncols
                                  ? __ldg(reinterpret_cast<const float4*>(col_sc + g.n_out + n0 + 4 * q4))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            u[4 * q4] *= rs * cs.x; u[4 * q4 + 1] *= rs * cs.y;
            u[4 * q4 + 2] *= rs * cs.z; u[4 * q4 + 3] *= rs * cs.w;
          }
        }
        bulk_wait_read();  // this thread's earlier copies have read the staging area ...
        __syncwarp();      // ... and so have the other lanes'
        if (p_ok) {
#pragma unroll
          for (int j8 = 0; j8 < 4; ++j8) {
            if (8 * j8 >= ncols) break;
            float* vv = v + 8 * j8;
            if (act_bwd) {  // [g A | dH (gate) | dH up] or [g A | dH]
              float a8[8], ga[8], dh[8], du[8], hg[8], hu[8];
              unpack8(ra[j8], a8);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                dg_acc = fmaf(vv[j], a8[j], dg_acc);
                ga[j] = gate * a8[j];
              }
              *chunk(0, j8) = pack8(ga);
              if (!g.out) continue;
              if (swi) {
                unpack8(rg[j8], hg);
                unpack8(ru[j8], hu);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float da = gate * vv[j];
                  const float sg = fast_sigmoid(hg[j]);
                  dh[j] = da * hu[j] * sg * fmaf(hg[j], 1.0f - sg, 1.0f);
                  du[j] = da * hg[j] * sg;
                }
                *chunk(1, j8) = pack8(dh);
                *chunk(2, j8) = pack8(du);
              } else {
                if (g.act == SMOE_ACT_GELU_TANH) {
                  unpack8(rg[j8], hg);
#pragma unroll
                  for (int j = 0; j < 8; ++j) dh[j] = gate * vv[j] * fast_gelu_grad(hg[j]);
                } else {
#pragma unroll
                  for (int j = 0; j < 8; ++j) dh[j] = gate * vv[j];
                }
                *chunk(1, j8) = pack8(dh);
              }
            } else if (epi_store) {  // [g acc]
              float o[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) o[j] = gate * vv[j];
              if (direct)
                *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(g.out) + (size_t)orow * g.ldo + n0 + 8 * j8) = pack8(o);
              else
                *chunk(0, j8) = pack8(o);
            } else {  // EPI_ACT_FWD: [H (gate) | H up | A] or [H | A]
              float a8[8];
              if (SWIGLU_FWD) {
                float* uu = u + 8 * j8;
#pragma unroll
                for (int j = 0; j < 8; ++j) a8[j] = vv[j] * fast_sigmoid(vv[j]) * uu[j];
                *chunk(0, j8) = pack8(vv);
                *chunk(1, j8) = pack8(uu);
                *chunk(2, j8) = pack8(a8);
              } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) a8[j] = fast_gelu(vv[j]);
                *chunk(0, j8) = pack8(vv);
                *chunk(1, j8) = pack8(a8);
              }
            }
          }
        }
        fence_proxy_async();  // the staged bytes are visible to the TMA engine
        __syncwarp();
        if (boxed) {
          if (lane == 0) {
            if (act_bwd) {
              if (g.out2) tma_store_3d(&tmO2, wstage_s, n0, 0, wrow0);
              if (g.out) {
                tma_store_3d(&tmO, wstage_s + kBoxBytes, n0, 0, wrow0);
                if (swi) tma_store_3d(&tmO, wstage_s + 2 * kBoxBytes, n0, 1, wrow0);
              }
            } else if (epi_store) {
              tma_store_3d(&tmO, wstage_s + kb * kBoxBytes, n0, 0, wrow0);
            } else {
              tma_store_3d(&tmO, wstage_s, n0, 0, wrow0);
              if (SWIGLU_FWD) {
                tma_store_3d(&tmO, wstage_s + kBoxBytes, n0, 1, wrow0);
                tma_store_3d(&tmO2, wstage_s + 2 * kBoxBytes, n0, 0, wrow0);
              } else {
                tma_store_3d(&tmO2, wstage_s + kBoxBytes, n0, 0, wrow0);
              }
            }
            bulk_commit();
          }
        } else if (p_ok && !direct) {
          if (act_bwd) {
            if (g.out2) bulk_s2g(reinterpret_cast<bf16*>(g.out2) + (size_t)i * g.ldo2 + n0, slot_s, seg);
            if (g.out) {
              if (swi) {
                bf16* O = reinterpret_cast<bf16*>(g.out) + (size_t)orow * g.ldo;
                bulk_s2g(O + n0, slot_s + 64, seg);
                bulk_s2g(O + g.n_out + n0, slot_s + 128, seg);
              } else {
                bulk_s2g(reinterpret_cast<bf16*>(g.out) + (size_t)orow * g.ldo + n0, slot_s + 64, seg);
              }
            }
          } else if (epi_store) {
            bulk_s2g(reinterpret_cast<bf16*>(g.out) + (size_t)orow * g.ldo + n0, slot_s, seg);
          } else {
            bf16* H = reinterpret_cast<bf16*>(g.out) + (size_t)orow * g.ldo;
            bf16* A2 = reinterpret_cast<bf16*>(g.out2) + (size_t)orow * g.ldo2;
            bulk_s2g(H + n0, slot_s, seg);
            if (SWIGLU_FWD) {
              bulk_s2g(H + g.n_out + n0, slot_s + 64, seg);
              bulk_s2g(A2 + n0, slot_s + 128, seg);
            } else {
              bulk_s2g(A2 + n0, slot_s + 64, seg);
            }
          }
          bulk_commit();
        }
      }
      if (act_bwd && p_ok && g.dg_partial)
        g.dg_partial[(size_t)i * g.dg_ld + t.nb] = dg_acc;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // the accumulator buffer is free (a pair: at the leader)
        if (PAIR && rank == 1) mbar_arrive_cluster(peer_addr(&c.tempty[buf], 0));
        else mbar_arrive(&c.tempty[buf]);
      }
    }
    bulk_wait_all();
  }
  teardown<PAIR>(c);
}

// ---------------------------------------------------------------------------
// dW kernel
// ---------------------------------------------------------------------------
// Gather of NS 64-column slabs of BK scattered rows (the MN-major operand of the
// dW product) with cp.async: thread t copies chunk (t % 8NS) of rows
// t / 8NS + (128 / 8NS) j.  The source rows come from a shared-memory ring that
// the index warp fills (slot -> row, range-checked) ahead of time; destination
// offsets are fixed per thread, so a copy costs a shared load, one address
// computation and the cp.async.  Rows marked -1 and columns past `ncols` are
// zero-filled.
template <int NS>
struct SlabGather {
  static constexpr int CPR = 8 * NS;
  static constexpr int RSTEP = kDwGatherThreads / CPR;
  static constexpr int NR = BK / RSTEP;
  int row0;        // first row of this thread
  uint32_t off0;   // shared-memory offset of (row0, chunk) inside a stage
  int chunk_col;   // column of this thread's chunk inside the tile

  __device__ __forceinline__ void init(int t) {
    const int cg = t % CPR, slab = cg >> 3, cc = cg & 7;
    row0 = t / CPR;
    off0 = slab * 8192 + sw128_off(row0, cc);
    chunk_col = 64 * slab + 8 * cc;
  }
  // rows row0 + RSTEP*j keep the same (row & 7) pattern only when RSTEP % 8 == 0;
  // otherwise the swizzled offset is recomputed per row.
  __device__ __forceinline__ uint32_t dst_off(int j, int t) const {
    if (RSTEP % 8 == 0) return off0 + (uint32_t)(RSTEP * j * 128);
    const int cg = t % CPR, slab = cg >> 3, cc = cg & 7;
    return slab * 8192 + sw128_off(row0 + RSTEP * j, cc);
  }
  __device__ __forceinline__ void issue(uint32_t dst, const int* rows, const bf16* base, int ld,
                                        int col0, int ncols, int t) const {
    const int col = col0 + chunk_col;
    const bool col_ok = col < ncols;
    const bf16* cbase = base + col;
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      const int sr = rows[row0 + RSTEP * j];
      const bool ok = col_ok && sr >= 0;
      cp_async16(dst + dst_off(j, t), ok ? cbase + (size_t)sr * ld : base, ok ? 16u : 0u);
    }
  }
  // This thread's gates of a stage (one per row it copies), from the index ring.
  __device__ __forceinline__ void load_gates(const float* gsc, float* g) const {
#pragma unroll
    for (int j = 0; j < NR; ++j) g[j] = gsc[row0 + RSTEP * j];
  }
  // Multiplies the chunks this thread copied into `stage` (already landed) by
  // their rows' gates: bf16 value times fp32 gate, rounded once to bf16.
  __device__ __forceinline__ void scale(uint8_t* stage, const float* g, int t) const {
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      uint4* p = reinterpret_cast<uint4*>(stage + dst_off(j, t));
      float v[8];
      unpack8(*p, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] *= g[j];
      *p = pack8(v);
    }
  }
};

// Gated gather of the A operand with deferred hand-over.  The gate multiplies the
// copied bytes in shared memory, so a stage can only be handed to the tensor core
// once this thread's copies of it have landed: each thread keeps its last kDefer
// stages in flight (one cp.async group per stage) and, after issuing a stage,
// waits for the group kDefer stages older, scales that stage's rows, makes the
// writes visible to the tensor core's (async) proxy and arrives on its full
// barrier.  kDefer < the ring depth, so the thread never waits on a stage that
// can only be freed by the hand-over it is holding back.
constexpr int kDefer = 2;
struct GatePending {
  int stage[kDefer + 1];
  bool live[kDefer + 1];
  float g[kDefer + 1][SlabGather<2>::NR];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i <= kDefer; ++i) live[i] = false;
  }
};
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// After the copies of `stage_idx` were issued (gates g_new): commit them as one
// group, then hand over the stage issued kDefer steps ago, if any.
__device__ __forceinline__ void gated_push(GatePending& q, const SlabGather<2>& ga, int t, int stage_idx,
                                           const float* g_new, uint8_t* ring, int stage_bytes,
                                           uint64_t* full) {
  cp_async_commit();
  q.stage[kDefer] = stage_idx;
  q.live[kDefer] = true;
#pragma unroll
  for (int j = 0; j < SlabGather<2>::NR; ++j) q.g[kDefer][j] = g_new[j];
  if (q.live[0]) {
    cp_async_wait_group<kDefer>();
    ga.scale(ring + q.stage[0] * stage_bytes, q.g[0], t);
    fence_proxy_async();
    mbar_arrive(&full[q.stage[0]]);
  }
#pragma unroll
  for (int i = 0; i < kDefer; ++i) {
    q.stage[i] = q.stage[i + 1];
    q.live[i] = q.live[i + 1];
#pragma unroll
    for (int j = 0; j < SlabGather<2>::NR; ++j) q.g[i][j] = q.g[i + 1][j];
  }
  q.live[kDefer] = false;
}
// Hands over every stage still held back (end of the work list).
__device__ __forceinline__ void gated_drain(GatePending& q, const SlabGather<2>& ga, int t, uint8_t* ring,
                                            int stage_bytes, uint64_t* full) {
  cp_async_wait_group<0>();
#pragma unroll
  for (int i = 0; i < kDefer; ++i) {
    if (!q.live[i]) continue;
    ga.scale(ring + q.stage[i] * stage_bytes, q.g[i], t);
    fence_proxy_async();
    mbar_arrive(&full[q.stage[i]]);
    q.live[i] = false;
  }
}

// The tile list of the dW kernels: a tile's work grows with its expert's rows, and
// routing can be very uneven, so the list runs over the experts from the most rows
// to the fewest and the P workers (CTAs, or CTA pairs) take it in rounds of P
// tiles, alternately forward and backward (every role derives the same sequence).
// Tile L -> (e, nb, mb), mb fastest.
struct DwTiles {
  int P, w;    // workers and this worker's index
  int nM, nN;  // M and N tiles per expert
  int total;
  __device__ __forceinline__ int tile(int j) const { return j * P + ((j & 1) ? P - 1 - w : w); }
  __device__ __forceinline__ void coords(const DwExtra& x, int L, int& e, int& mb, int& nb) const {
    e = x.order[L / (nM * nN)];
    const int rem = L % (nM * nN);
    nb = rem / nM;
    mb = rem % nM;
  }
};

// Experts by descending row count (ties: lower id); with more than 256 experts
// the tiles keep the expert index order.  Ends with a block barrier.
__device__ __forceinline__ void dw_expert_order(DwExtra& x, int E) {
  if (E <= 256) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      const int n = x.off[e + 1] - x.off[e];
      int rank = 0;
      for (int f = 0; f < E; ++f) {
        const int m = x.off[f + 1] - x.off[f];
        rank += (m > n) || (m == n && f < e);
      }
      x.order[rank] = (short)e;
    }
  } else {
    for (int e = threadIdx.x; e < E; e += blockDim.x) x.order[e] = (short)e;
  }
  __syncthreads();
}

// Walks the (tile, K-block) stages of a dW worker's tile list in order.
struct DwStageIt {
  int jt, L, rb, re, nK, kb;
  bool valid;
  // From tile L at K-block kb (0 for a new tile): skip tiles without rows.
  __device__ __forceinline__ void settle(const DwTiles& tl, const DwExtra& x) {
    while (L < tl.total) {
      int e, mb, nb;
      tl.coords(x, L, e, mb, nb);
      rb = x.off[e];
      re = x.off[e + 1];
      nK = cdiv(re - rb, BK);
      if (kb < nK) { valid = true; return; }
      L = tl.tile(++jt);
      kb = 0;
    }
    valid = false;
    nK = 0;
  }
  __device__ __forceinline__ void init(const DwTiles& tl, const DwExtra& x) {
    jt = 0;
    L = tl.tile(0);
    kb = 0;
    settle(tl, x);
  }
  // The tile's coordinates are derived again only when its K-blocks run out.
  __device__ __forceinline__ void next(const DwTiles& tl, const DwExtra& x) {
    if (++kb < nK) return;
    L = tl.tile(++jt);
    kb = 0;
    settle(tl, x);
  }
};

// Source-row producer of the dW gathers (one warp).  The slot ids of kIdxBatch
// stages are loaded together, and those of the next batch are already in flight
// while this batch is written to the ring, so the global-load latency overlaps
// the wait for free ring slots instead of stalling the gathers.  Each slot p
// becomes the source row p / fan_out (a shift for a power of two), checked
// against the operand's row count; -1 marks a zero row.  A_SCALE: the slot's gate
// goes beside it, and a grouped A (gathered row by row) takes grouped row r itself.
template <bool A_GATHER, bool B_GATHER, bool A_SCALE>
__device__ __forceinline__ void dw_index_producer(SharedCtl& c, DwExtra& x, const DwGemm& g,
                                                  const DwTiles& tl, volatile int* abort_flag, int lane) {
  constexpr int kIdxBatch = IDX_STAGES / 2;
  constexpr int NQ = BK / 32;  // slots per lane per stage
  const int a_shift = (g.a_fan_out & (g.a_fan_out - 1)) == 0 ? __ffs(g.a_fan_out) - 1 : -1;
  const int b_shift = (g.b_fan_out & (g.b_fan_out - 1)) == 0 ? __ffs(g.b_fan_out) - 1 : -1;
  auto src_of = [&](int p, int shift, int fan, int rows) -> int {
    if (p < 0) return -1;
    const int r = shift >= 0 ? (p >> shift) : p / fan;
    if (r >= rows) {
      report_error(g.err, ERRBIT_DATA);
      return -1;
    }
    return r;
  };
  const bool a_ident = g.a_mode == ROWS_GROUPED;
  // slot ids of the next kIdxBatch stages of `it` (-1 past a slice end)
  auto load_batch = [&](DwStageIt& it, int (&v)[kIdxBatch][NQ], int (&r0)[kIdxBatch]) {
#pragma unroll
    for (int b = 0; b < kIdxBatch; ++b) {
      r0[b] = it.valid ? it.rb + it.kb * BK : 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int r = r0[b] + lane + 32 * q;
        v[b][q] = (it.valid && r < it.re) ? __ldg(g.sorted_slot + r) : -1;
      }
      if (it.valid) it.next(tl, x);
    }
  };
  DwStageIt ld, wr;
  ld.init(tl, x);
  wr = ld;
  int va[kIdxBatch][NQ], ra[kIdxBatch];
  load_batch(ld, va, ra);
  Ring ri;
  while (wr.valid) {
    int vb[kIdxBatch][NQ], rbn[kIdxBatch];
    load_batch(ld, vb, rbn);  // the next batch, in flight while this one is written
    float gv[kIdxBatch][NQ];
#pragma unroll
    for (int b = 0; b < kIdxBatch; ++b)
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        gv[b][q] = 0.0f;
        if (A_SCALE) {
          const int p = va[b][q];
          if (p >= 0 && p < g.num_rows) gv[b][q] = __ldg(g.row_gates + p);
        }
      }
    bool run = true;
#pragma unroll
    for (int b = 0; b < kIdxBatch; ++b) {
      if (!wr.valid) break;
      if (!mbar_wait(&c.iempty[ri.s], ri.ph ^ 1, abort_flag, g.err)) { run = false; break; }
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int r = ra[b] + lane + 32 * q;
        if (A_GATHER) {
          int a_src;
          if (a_ident) a_src = (va[b][q] < 0 || r >= g.a_rows) ? -1 : r;  // grouped A, gathered by row
          else a_src = src_of(va[b][q], a_shift, g.a_fan_out, g.a_rows);
          x.idx[ri.s][0][lane + 32 * q] = a_src;
        }
        if (A_SCALE) x.gsc[ri.s][lane + 32 * q] = gv[b][q];
        if (B_GATHER) x.idx[ri.s][1][lane + 32 * q] = src_of(va[b][q], b_shift, g.b_fan_out, g.b_rows);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.ifull[ri.s]);
      ri.next(IDX_STAGES);
      wr.next(tl, x);
    }
    if (!run) break;
#pragma unroll
    for (int b = 0; b < kIdxBatch; ++b) {
      ra[b] = rbn[b];
#pragma unroll
      for (int q = 0; q < NQ; ++q) va[b][q] = vb[b][q];
    }
  }
}

// Epilogue of a dW tile: this warp's 32 accumulator rows (M = m0 + 32 q + lane)
// times the tile's BN columns (from n0), from tensor memory (zeros when the
// expert has no rows).  d_boxed: per 32-column chunk the warp writes its 32 x 32
// fp32 block into a 128-byte-swizzled box (transposed for TRANS_OUT) that one TMA
// tensor store writes out, clipped to dW's bounds; else plain stores.
template <bool TRANS_OUT>
__device__ __forceinline__ void dw_store_tile(const DwGemm& g, const CUtensorMap* tmD, int d_boxed,
                                              uint8_t* box, uint32_t box_s, uint32_t trow,
                                              bool has_rows, int e, int m0, int n0, int q, int lane) {
  const int m = m0 + q * 32 + lane;
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 32) {
    float v[32];
    if (has_rows) {
      tmem_ld32(trow + c0, v);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.0f;
    }
    if (d_boxed) {
      if (n0 + c0 >= g.N) break;  // warp-uniform
      if (lane == 0) bulk_wait_read();  // the previous chunk's store has read the box
      __syncwarp();
      if (TRANS_OUT) {  // box[n][m]: row j = column n, lane = m
#pragma unroll
        for (int j = 0; j < 32; ++j)
          *reinterpret_cast<float*>(box + j * 128 + ((((lane >> 2) ^ (j & 7))) << 4) + ((lane & 3) << 2)) = v[j];
      } else {  // box[m][n]: row lane = m
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4)
          *reinterpret_cast<float4*>(box + lane * 128 + ((j4 ^ (lane & 7)) << 4)) =
              make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        if (TRANS_OUT) tma_store_3d(tmD, box_s, m0 + q * 32, n0 + c0, e);
        else tma_store_3d(tmD, box_s, n0 + c0, m0 + q * 32, e);
        bulk_commit();
      }
      continue;
    }
    if (m >= g.M) continue;
    if (TRANS_OUT) {  // dW[e][n][m]: lanes hold consecutive m -> 128-byte lines
      float* out = g.dw + (size_t)e * g.N * g.M + m;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int n = n0 + c0 + j;
        if (n < g.N) out[(size_t)n * g.M] = v[j];
      }
    } else {
      float* out = g.dw + ((size_t)e * g.M + m) * g.N;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const int n = n0 + c0 + 4 * j4;
        if (n >= g.N) break;
        *reinterpret_cast<float4*>(out + n) =
            make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
      }
    }
  }
}

// dW[e] tile (e, m-block, n-block) of D[m, n] = sum over the expert's rows r of
// A[r, m] * B[r, n].  TRANS_OUT stores D transposed (the host swapped the
// operands so that a gathered operand sits on the 128-wide A side); the store
// is then coalesced across the warp (consecutive m, one n at a time).
// A_SCALE: A is gathered (through sorted_slot, or row by row when it is grouped)
// and each of its rows is multiplied by the gate of its slot on the way in.
template <bool A_GATHER, bool B_GATHER, bool TRANS_OUT, bool A_SCALE = false>
__global__ void __launch_bounds__(kDwThreads, 1)
dw_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmD, const DwGemm g, int nM, int nN,
                  int d_boxed, int slabs) {
  // four stages of each operand (16 KB A + 32 KB B): a deeper A ring for the gather
  // at the cost of a 3-stage B ring measured about 1% slower.  The two rings advance
  // together, so one empty barrier per stage (emptyA) frees both: one MMA commit per
  // stage instead of two.
  constexpr int SA = 4, SB = 4;
  static_assert(SA == SB, "the A and B rings share their empty barriers");
  static_assert(SA * A_BYTES + SB * B_BYTES <= kRingBytes, "stage rings exceed their budget");
  static_assert(!A_SCALE || (A_GATHER && kDefer < SA), "gated rows are gathered, deferred < ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + SA * A_BYTES;
  SharedCtl& c = *reinterpret_cast<SharedCtl*>(smem + kRingBytes);
  DwExtra& x = *reinterpret_cast<DwExtra*>(smem + kRingBytes + kCtlBytes);
  volatile int* abort_flag = &c.abort_flag;

  setup<SA, SB>(c, g.offsets, g.E, g.num_rows, g.err, A_GATHER ? kDwGatherThreads : 1,
                B_GATHER ? kDwGatherThreads : 1, kDwGatherThreads / 32, x.off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool offsets_ok = c.total_mtiles > 0 || g.num_rows == 0;
  DwTiles tl;
  tl.P = (int)gridDim.x;
  tl.w = (int)blockIdx.x;
  tl.nM = nM;
  tl.nN = nN;
  tl.total = offsets_ok ? g.E * nM * nN : 0;
  dw_expert_order(x, g.E);

  if (warp == 0) {
    // ---------------- TMA producer of the grouped operand(s) ----------------
    if (lane == 0 && !(A_GATHER && B_GATHER)) {
      Ring ra, rb;
      bool run = true;
      for (int jt = 0, L = tl.tile(0); run && L < tl.total; L = tl.tile(++jt)) {
        int e, mb, nb;
        tl.coords(x, L, e, mb, nb);
        const int r_begin = x.off[e], r_end = x.off[e + 1];
        const int nK = cdiv(r_end - r_begin, BK);
        for (int kb = 0; kb < nK; ++kb) {
          const int rk = r_begin + kb * BK;
          if (!A_GATHER) {  // 64 rows x 128 M-columns: two 64-column slabs of 8 KB
            if (!mbar_wait(&c.emptyA[ra.s], ra.ph ^ 1, abort_flag, g.err)) { run = false; break; }
            uint8_t* a_dst = sA + ra.s * A_BYTES;
            mbar_expect_tx(&c.fullA[ra.s], A_BYTES);
            if (slabs & 1) {  // slab view {64, rows, slabs}: both slabs in one load
              tma_load_3d(a_dst, &tmA, &c.fullA[ra.s], 0, rk, mb * (BM / 64));
            } else {
              tma_load_2d(a_dst, &tmA, &c.fullA[ra.s], mb * BM, rk);
              tma_load_2d(a_dst + 8192, &tmA, &c.fullA[ra.s], mb * BM + 64, rk);
            }
            ra.next(SA);
          }
          if (!B_GATHER) {  // 64 rows x 256 N-columns: four slabs
            if (!mbar_wait(&c.emptyA[rb.s], rb.ph ^ 1, abort_flag, g.err)) { run = false; break; }
            uint8_t* b_dst = sB + rb.s * B_BYTES;
            mbar_expect_tx(&c.fullB[rb.s], B_BYTES);
            if (slabs & 2) {  // slab view: the four slabs in one load
              tma_load_3d(b_dst, &tmB, &c.fullB[rb.s], 0, rk, nb * (BN / 64));
            } else {
#pragma unroll
              for (int slab = 0; slab < 4; ++slab)
                tma_load_2d(b_dst + slab * 8192, &tmB, &c.fullB[rb.s], nb * BN + 64 * slab, rk);
            }
            rb.next(SB);
          }
        }
      }
    }
    __syncwarp();
  } else if ((A_GATHER || B_GATHER) && warp == 2) {
    // ---------------- source-row producer for the gathers ----------------
    dw_index_producer<A_GATHER, B_GATHER, A_SCALE>(c, x, g, tl, abort_flag, lane);
  } else if ((A_GATHER || B_GATHER) && warp >= kGatherWarp0 &&
             warp < kGatherWarp0 + kDwGatherThreads / 32) {
    // ---------------- cp.async gather of the scattered operand(s) ----------------
    const int t = threadIdx.x - kGatherWarp0 * 32;
    SlabGather<2> ga;
    SlabGather<4> gb;
    ga.init(t);
    gb.init(t);
    GatePending pend;
    pend.init();
    Ring ra, rb, ri;
    bool run = true;
    for (int jt = 0, L = tl.tile(0); run && L < tl.total; L = tl.tile(++jt)) {
      int e, mb, nb;
      tl.coords(x, L, e, mb, nb);
      const int nK = cdiv(x.off[e + 1] - x.off[e], BK);
      for (int kb = 0; kb < nK; ++kb) {
        if (!mbar_wait(&c.ifull[ri.s], ri.ph, abort_flag, g.err)) { run = false; break; }
        if (A_GATHER) {
          if (!mbar_wait(&c.emptyA[ra.s], ra.ph ^ 1, abort_flag, g.err)) { run = false; break; }
          ga.issue(smem_u32(sA + ra.s * A_BYTES), x.idx[ri.s][0], reinterpret_cast<const bf16*>(g.a),
                   g.lda, mb * BM, g.M, t);
          if (A_SCALE) {
            float gn[SlabGather<2>::NR];
            ga.load_gates(x.gsc[ri.s], gn);
            gated_push(pend, ga, t, ra.s, gn, sA, A_BYTES, c.fullA);
          } else {
            cp_async_arrive(&c.fullA[ra.s]);
          }
          ra.next(SA);
        }
        if (B_GATHER) {
          if (!mbar_wait(&c.emptyA[rb.s], rb.ph ^ 1, abort_flag, g.err)) { run = false; break; }
          gb.issue(smem_u32(sB + rb.s * B_BYTES), x.idx[ri.s][1], reinterpret_cast<const bf16*>(g.b),
                   g.ldb, nb * BN, g.N, t);
          cp_async_arrive(&c.fullB[rb.s]);
          rb.next(SB);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.iempty[ri.s]);  // this warp is done with the rows
        ri.next(IDX_STAGES);
      }
    }
    if (A_SCALE && run) gated_drain(pend, ga, t, sA, A_BYTES, c.fullA);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // With a gathered operand its rows past the slice are zero-filled, so the
    // other operand's rows there (finite data or zero fill) contribute nothing and
    // one lane runs the loop.  With two grouped operands the warp zeroes the
    // tail rows of both in shared memory first.
    constexpr bool kGather = A_GATHER || B_GATHER;
    constexpr uint32_t idesc = idesc_bf16(BM, BN, 1, 1);
    if (!kGather || lane == 0) {
      Ring ra, rb;
      int it = 0;
      for (int jt = 0, L = tl.tile(0); L < tl.total; L = tl.tile(++jt), ++it) {
        int e, mb, nb;
        tl.coords(x, L, e, mb, nb);
        const int r_begin = x.off[e], r_end = x.off[e + 1];
        const int nK = cdiv(r_end - r_begin, BK);
        const int buf = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!mbar_wait(&c.tempty[buf], tph ^ 1, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = c.tmem_base + buf * BN;
        bool ok = true;
        for (int kb = 0; kb < nK; ++kb) {
          if (!mbar_wait(&c.fullA[ra.s], ra.ph, abort_flag, g.err) ||
              !mbar_wait(&c.fullB[rb.s], rb.ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          if (kGather) {
            fence_proxy_async();  // cp.async rows -> tensor core
          } else {
            const int valid = min(BK, r_end - (r_begin + kb * BK));
            if (valid < BK) {  // rows past the slice end hold other rows' data
              uint8_t* a_t = sA + ra.s * A_BYTES;
              uint8_t* b_t = sB + rb.s * B_BYTES;
              const int nz = (BK - valid) * 8;  // 16-byte chunks per slab
              for (int z = lane; z < nz * 6; z += 32) {
                const int slab = z / nz, w = z % nz;
                uint8_t* base = slab < 2 ? a_t + slab * 8192 : b_t + (slab - 2) * 8192;
                *reinterpret_cast<uint4*>(base + valid * 128 + w * 16) = make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async();
            }
            __syncwarp();
          }
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(sA + ra.s * A_BYTES);
            const uint32_t b_addr = smem_u32(sB + rb.s * B_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_bf16(d_tmem, desc_mnmajor(a_addr + kk * 2048), desc_mnmajor(b_addr + kk * 2048),
                        idesc, (kb | kk) != 0);
            umma_commit(&c.emptyA[ra.s]);  // frees the stage of both rings
          }
          if (!kGather) __syncwarp();
          ra.next(SA);
          rb.next(SB);
        }
        if (!ok) break;
        if (lane == 0) {
          if (nK > 0) umma_commit(&c.tfull[buf]);
          else mbar_arrive(&c.tfull[buf]);
        }
        if (!kGather) __syncwarp();
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ---------------- epilogue: one accumulator row per thread ----------------
    const int q = warp - 4;
    uint8_t* box = smem + kRingBytes + kCtlBytes + kDwExtraBytes + q * kDwBoxBytes;
    const uint32_t box_s = smem_u32(box);
    int it = 0;
    for (int jt = 0, L = tl.tile(0); L < tl.total; L = tl.tile(++jt), ++it) {
      int e, mb, nb;
      tl.coords(x, L, e, mb, nb);
      const int nrows = x.off[e + 1] - x.off[e];
      const int buf = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (!mbar_wait(&c.tfull[buf], tph, abort_flag, g.err)) break;
      tc_fence_after();
      const uint32_t trow = c.tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
      dw_store_tile<TRANS_OUT>(g, &tmD, d_boxed, box, box_s, trow, nrows > 0, e, mb * BM, nb * BN, q, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.tempty[buf]);
    }
    if (lane == 0) bulk_wait_all();
  }
  teardown(c);
}

// ---------------------------------------------------------------------------
// dW kernel on CTA pairs (cta_group::2)
// ---------------------------------------------------------------------------
// A cluster of two CTAs takes a 256 (M) x 256 (N) tile of dW[e] with M = 256
// MMAs.  For the same 64 slice rows per stage, CTA r gathers M columns
// [128 r, 128 r + 128) of the tile's A rows (the scattered operand, optionally
// gated) and TMA-loads N columns [128 r, 128 r + 128) of B, so a CTA brings 32 KB
// per K-block instead of 48 KB and its ring holds six stages instead of four:
// about 2.5x the single-CTA kernel's look-ahead in time, which is what the
// gather's latency needs.  Rank 0 issues the MMAs once its own stage has landed
// (its gathered rows, plus both CTAs' TMA bytes, which count on its barrier) and
// rank 1 has relayed that its gathered rows have landed; it commits to both
// CTAs' empty barriers.  Each CTA's tensor memory holds its 128 rows of the
// accumulator (all 256 columns), drained by its own epilogue warps; rank 1's
// epilogue frees an accumulator buffer on rank 0's barrier.  No load uses
// multicast: every CTA fetches its own bytes.
template <bool A_SCALE, bool TRANS_OUT>
__global__ void __launch_bounds__(kDwThreads, 1)
dw_pair_tc_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmD,
                  const DwGemm g, int nMP, int nN, int d_boxed, int slabs) {
  constexpr int STAGES = 6;
  constexpr int BH = B_BYTES / 2;  // this CTA's half of B per stage (16 KB)
  static_assert(STAGES * (A_BYTES + BH) <= kRingBytes && STAGES <= kMaxStages && kDefer < STAGES,
                "pair ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  SharedCtl& c = *reinterpret_cast<SharedCtl*>(smem + kRingBytes);
  DwExtra& x = *reinterpret_cast<DwExtra*>(smem + kRingBytes + kCtlBytes);
  volatile int* abort_flag = &c.abort_flag;
  const int rank = (int)cluster_rank();
  // a stage's full barrier: this CTA's gather threads, plus at rank 0 the
  // producer's expect-tx for both CTAs' B halves
  setup<STAGES, 0, true>(c, g.offsets, g.E, g.num_rows, g.err,
                         (uint32_t)kDwGatherThreads + (rank == 0 ? 1u : 0u), 1, kDwGatherThreads / 32,
                         x.off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool offsets_ok = c.total_mtiles > 0 || g.num_rows == 0;
  DwTiles tl;
  tl.P = (int)(gridDim.x >> 1);
  tl.w = (int)(blockIdx.x >> 1);
  tl.nM = nMP;
  tl.nN = nN;
  tl.total = offsets_ok ? g.E * nMP * nN : 0;
  dw_expert_order(x, g.E);

  if (warp == 0) {
    // ---------------- TMA producer: this CTA's half of the B columns ----------------
    if (lane == 0) {
      Ring r;
      bool run = true;
      for (int jt = 0, L = tl.tile(0); run && L < tl.total; L = tl.tile(++jt)) {
        int e, mp, nb;
        tl.coords(x, L, e, mp, nb);
        const int r_begin = x.off[e], r_end = x.off[e + 1];
        const int nK = cdiv(r_end - r_begin, BK);
        for (int kb = 0; kb < nK; ++kb) {
          if (!mbar_wait(&c.emptyA[r.s], r.ph ^ 1, abort_flag, g.err)) { run = false; break; }
          const uint32_t full_cl = peer_addr(&c.fullA[r.s], 0);
          if (rank == 0) mbar_expect_tx(&c.fullA[r.s], 2 * BH);
          uint8_t* b_dst = sB + r.s * BH;
          const int col = nb * BN + rank * (BN / 2);
          if (slabs & 2) {  // slab view: this CTA's two slabs in one load
            tma_load_3d_pair(b_dst, &tmB, full_cl, 0, r_begin + kb * BK, col / 64);
          } else {
            tma_load_2d_pair(b_dst, &tmB, full_cl, col, r_begin + kb * BK);
            tma_load_2d_pair(b_dst + 8192, &tmB, full_cl, col + 64, r_begin + kb * BK);
          }
          r.next(STAGES);
        }
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------- source-row producer (both CTAs build the same rows) ----------------
    dw_index_producer<true, false, A_SCALE>(c, x, g, tl, abort_flag, lane);
  } else if (warp >= kGatherWarp0 && warp < kGatherWarp0 + kDwGatherThreads / 32) {
    // ---------------- cp.async gather of this CTA's 128 A columns ----------------
    const int t = threadIdx.x - kGatherWarp0 * 32;
    SlabGather<2> ga;
    ga.init(t);
    GatePending pend;
    pend.init();
    Ring r, ri;
    bool run = true;
    for (int jt = 0, L = tl.tile(0); run && L < tl.total; L = tl.tile(++jt)) {
      int e, mp, nb;
      tl.coords(x, L, e, mp, nb);
      const int nK = cdiv(x.off[e + 1] - x.off[e], BK);
      for (int kb = 0; kb < nK; ++kb) {
        if (!mbar_wait(&c.ifull[ri.s], ri.ph, abort_flag, g.err)) { run = false; break; }
        if (!mbar_wait(&c.emptyA[r.s], r.ph ^ 1, abort_flag, g.err)) { run = false; break; }
        ga.issue(smem_u32(sA + r.s * A_BYTES), x.idx[ri.s][0], reinterpret_cast<const bf16*>(g.a), g.lda,
                 mp * 2 * BM + rank * BM, g.M, t);
        if (A_SCALE) {
          float gn[SlabGather<2>::NR];
          ga.load_gates(x.gsc[ri.s], gn);
          gated_push(pend, ga, t, r.s, gn, sA, A_BYTES, c.fullA);
        } else {
          cp_async_arrive(&c.fullA[r.s]);
        }
        r.next(STAGES);
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.iempty[ri.s]);
        ri.next(IDX_STAGES);
      }
    }
    if (A_SCALE && run) gated_drain(pend, ga, t, sA, A_BYTES, c.fullA);
  } else if (warp == 1) {
    if (lane == 0 && rank == 1) {
      // ---------------- relay: this CTA's gathered rows of a stage have landed ----------------
      Ring r;
      bool run = true;
      for (int jt = 0, L = tl.tile(0); run && L < tl.total; L = tl.tile(++jt)) {
        int e, mp, nb;
        tl.coords(x, L, e, mp, nb);
        const int nK = cdiv(x.off[e + 1] - x.off[e], BK);
        for (int kb = 0; kb < nK; ++kb) {
          if (!mbar_wait(&c.fullA[r.s], r.ph, abort_flag, g.err)) { run = false; break; }
          fence_proxy_async();  // rows written by cp.async (and the gate pass), read by the tensor core
          mbar_arrive_cluster_relaxed(peer_addr(&c.pfull[r.s], 0));
          r.next(STAGES);
        }
      }
    } else if (lane == 0) {
      // ---------------- MMA issuer (rank 0) ----------------
      constexpr uint32_t idesc = idesc_bf16(2 * BM, BN, 1, 1);
      Ring r;
      int it = 0;
      for (int jt = 0, L = tl.tile(0); L < tl.total; L = tl.tile(++jt), ++it) {
        int e, mp, nb;
        tl.coords(x, L, e, mp, nb);
        const int nK = cdiv(x.off[e + 1] - x.off[e], BK);
        const int buf = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!mbar_wait(&c.tempty[buf], tph ^ 1, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = c.tmem_base + buf * BN;
        bool ok = true;
        for (int kb = 0; kb < nK; ++kb) {
          if (!mbar_wait(&c.fullA[r.s], r.ph, abort_flag, g.err) ||
              !mbar_wait(&c.pfull[r.s], r.ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          fence_proxy_async();  // rows written by cp.async (and the gate pass), read by the tensor core
          const uint32_t a_addr = smem_u32(sA + r.s * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + r.s * BH);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_pair(d_tmem, desc_mnmajor(a_addr + kk * 2048), desc_mnmajor(b_addr + kk * 2048), idesc,
                           (kb | kk) != 0);
          umma_commit_pair_both(&c.emptyA[r.s]);  // the stage is free in both CTAs
          r.next(STAGES);
        }
        if (!ok) break;
        if (nK > 0) {
          umma_commit_pair_both(&c.tfull[buf]);
        } else {  // an empty expert: both epilogues write zeros
          mbar_arrive(&c.tfull[buf]);
          mbar_arrive_cluster(peer_addr(&c.tfull[buf], 1));
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ---------------- epilogue: this CTA's 128 accumulator rows ----------------
    const int q = warp - 4;
    uint8_t* box = smem + kRingBytes + kCtlBytes + kDwExtraBytes + q * kDwBoxBytes;
    const uint32_t box_s = smem_u32(box);
    int it = 0;
    for (int jt = 0, L = tl.tile(0); L < tl.total; L = tl.tile(++jt), ++it) {
      int e, mp, nb;
      tl.coords(x, L, e, mp, nb);
      const int nrows = x.off[e + 1] - x.off[e];
      const int buf = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (!mbar_wait(&c.tfull[buf], tph, abort_flag, g.err)) break;
      tc_fence_after();
      const uint32_t trow = c.tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
      dw_store_tile<TRANS_OUT>(g, &tmD, d_boxed, box, box_s, trow, nrows > 0, e, mp * 2 * BM + rank * BM,
                               nb * BN, q, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // the accumulator buffer is free (counted at rank 0)
        if (rank == 0) mbar_arrive(&c.tempty[buf]);
        else mbar_arrive_cluster(peer_addr(&c.tempty[buf], 0));
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  teardown<true>(c);
}

// ---------------------------------------------------------------------------
// Self-test of the failure path: the bounded wait on a barrier that nothing
// completes gives up after limit_ns and records the timeout.
// ---------------------------------------------------------------------------
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, unsigned* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches
// ---------------------------------------------------------------------------
// 2-D map over rows of a row-major [rows, cols] bf16 matrix with leading dimension ld.
cudaError_t rows_map(CUtensorMap* m, const void* base, int cols, int rows, int ld, uint32_t box_rows) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)(rows > 0 ? rows : 1)};
  const uint64_t strides[1] = {(uint64_t)ld * 2};
  const uint32_t box[2] = {64, box_rows};
  return make_map(m, base, 2, dims, strides, box);
}

// Slab view of [rows, ld] bf16 rows whose first `cols` columns (a multiple of 64)
// are used: dims {64, rows, cols / 64}, strides {ld * 2, 128}; a box is `nslab`
// slabs of 64 columns x box_rows rows, landing slab after slab (8 KB per 64 rows).
cudaError_t slab_map(CUtensorMap* m, const void* base, int cols, int rows, int ld, uint32_t box_rows,
                     uint32_t nslab) {
  if (cols % 64) return cudaErrorInvalidValue;
  const uint64_t dims[3] = {64, (uint64_t)(rows > 0 ? rows : 1), (uint64_t)cols / 64};
  const uint64_t strides[2] = {(uint64_t)ld * 2, 128};
  const uint32_t box[3] = {64, box_rows, nslab};
  return make_map(m, base, 3, dims, strides, box);
}

// Output map of the grouped epilogue's boxed stores: rows of [rows, ld] whose
// first parts * n_out columns hold `parts` blocks of n_out (SwiGLU's gate and up
// halves), as dims {n_out, parts, rows} so that a box never crosses n_out.
cudaError_t out_map(CUtensorMap* m, const void* base, int n_out, int parts, int rows, int ld) {
  const uint64_t dims[3] = {(uint64_t)n_out, (uint64_t)parts, (uint64_t)rows};
  const uint64_t strides[2] = {(uint64_t)n_out * 2, (uint64_t)ld * 2};
  const uint32_t box[3] = {32, 1, 32};
  return make_map(m, base, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

template <typename K>
cudaError_t prep(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

struct EpiMaps {
  CUtensorMap out{}, out2{}, xa{}, xh{};  // zero: unused maps are passed but never read
  int flags = 0;
};

// Persistent grid over `tiles` tiles: one CTA per SM, or for pairs as many
// 2-CTA clusters as the device can hold at once (fewer than half the SMs when a
// GPC has an odd number of free SMs; a cluster beyond that would run its whole
// share of the tile list after the others).
template <bool AG, bool BK_, bool SW, bool kPair = false, bool SPLIT = false, bool SHORT = false,
          bool F8 = false, bool G128 = false>
cudaError_t launch_g(const CUtensorMap& ta, const CUtensorMap& tb, const EpiMaps& m,
                     const GroupedGemm& g, int nN, long long tiles, cudaStream_t s) {
  static_assert(!kPair || !(SPLIT || SHORT || F8), "pairs: plain bf16 products");
  auto kern = grouped_gemm_tc_kernel<AG, BK_, SW, kPair, SPLIT, SHORT, F8, G128>;
  cudaError_t e = prep(kern, kGroupedSmem);
  if (e != cudaSuccess) return e;
  if (!kPair) {
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    kern<<<grid, kThreads, kGroupedSmem, s>>>(ta, tb, m.out, m.out2, m.xa, m.xh, g, nN, m.flags);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(num_sms() & ~1), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kGroupedSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters = 0;  // per instantiation
  if (max_clusters <= 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms() / 2;
    }
    max_clusters = n;
  }
  const long long pairs = tiles < max_clusters ? tiles : max_clusters;
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  e = cudaLaunchKernelEx(&cfg, kern, ta, tb, m.out, m.out2, m.xa, m.xh, g, nN, m.flags);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool AG, bool BG, bool TR, bool SC = false>
cudaError_t launch_d(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                     int d_boxed, int slabs, const DwGemm& g, int nM, int nN, int grid, cudaStream_t s) {
  auto kern = dw_gemm_tc_kernel<AG, BG, TR, SC>;
  cudaError_t e = prep(kern, kDwSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kDwThreads, kDwSmem, s>>>(ta, tb, td, g, nM, nN, d_boxed, slabs);
  return cudaGetLastError();
}

// The pair dW kernel on as many 2-CTA clusters as the device holds at once (at
// most one per tile pair).
template <bool SC, bool TR>
cudaError_t launch_dp(const CUtensorMap& tb, const CUtensorMap& td, int d_boxed, int slabs,
                      const DwGemm& g, int nMP, int nN, long long tiles, cudaStream_t s) {
  auto kern = dw_pair_tc_kernel<SC, TR>;
  cudaError_t e = prep(kern, kDwSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(num_sms() & ~1), 1, 1);
  cfg.blockDim = dim3(kDwThreads, 1, 1);
  cfg.dynamicSmemBytes = kDwSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters = 0;  // per instantiation
  if (max_clusters <= 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms() / 2;
    }
    max_clusters = n;
  }
  const long long pairs = tiles < max_clusters ? tiles : max_clusters;
  if (pairs <= 0) return cudaSuccess;
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  e = cudaLaunchKernelEx(&cfg, kern, tb, td, g, nMP, nN, d_boxed, slabs);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

namespace {
volatile int g_gemm_policy = 0;  // smoe_set_gemm_policy
}  // namespace

void set_gemm_policy(int policy) { g_gemm_policy = policy; }

bool tc_supported() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10 && encode_fn() != nullptr;
}

int tc_tile_cols() { return BN; }

int grouped_ksplit(int num_rows, int E, int n_out, int K, int fp8) {
  constexpr long long kSms = 148;  // a fixed count, so the split (and the workspace) is the same on any GPU
  const long long tiles = (long long)(cdiv(num_rows, BM) + (E < num_rows ? E : num_rows)) * cdiv(n_out, BN);
  if (tiles <= 0 || tiles * 2 > kSms) return 1;
  int ks = (int)((kSms + tiles - 1) / tiles);
  if (ks > 8) ks = 8;
  const int most = cdiv(K, fp8 ? 2 * BK : BK) / 4;  // at least four K-blocks per split
  if (ks > most) ks = most;
  return ks > 1 ? ks : 1;
}

// FP8 products (e4m3 codes, K-major weights): the up projection with a row gather
// and the activation epilogue, and the down projection (grouped rows, plain or
// split-K store).
cudaError_t launch_grouped_gemm_fp8(const GroupedGemm& g, cudaStream_t s) {
  const bool swiglu = g.epi == EPI_ACT_FWD && g.act == SMOE_ACT_SWIGLU;
  const int BNo = swiglu ? BN / 2 : BN;
  const int nN = cdiv(g.n_out, BNo);
  if (g.b_kn != 0 || !g.row_scale || !g.col_scale || g.epi == EPI_ACT_BWD) return cudaErrorInvalidValue;
  if (g.K % 16 || g.ksplit > cdiv(g.K, 2 * BK)) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  {  // A codes [a_rows, K] (grouped products): 128 x 128 boxes
    const uint64_t dims[2] = {(uint64_t)g.K, (uint64_t)(g.a_rows > 0 ? g.a_rows : 1)};
    const uint64_t str[1] = {(uint64_t)g.lda};
    const uint32_t box[2] = {128, (uint32_t)BM};
    cudaError_t e = make_map(&ta, g.a, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (e != cudaSuccess) return e;
  }
  {  // W codes [E, NW, K]: dims {K, NW, E}; SwiGLU loads its gate and up rows separately
    const uint64_t dims[3] = {(uint64_t)g.K, (uint64_t)g.NW, (uint64_t)g.E};
    const uint64_t str[2] = {(uint64_t)g.K, (uint64_t)g.NW * g.K};
    const uint32_t box[3] = {128, (uint32_t)(swiglu ? BN / 2 : BN), 1};
    cudaError_t e = make_map(&tb, g.b, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (e != cudaSuccess) return e;
  }
  EpiMaps m;
  const int parts = swiglu ? 2 : 1;
  bool st = g.out != nullptr && (g.out_mode == ROWS_GROUPED);
  if (st && out_map(&m.out, g.out, g.n_out, parts, g.num_rows, g.ldo) != cudaSuccess) st = false;
  if (st && g.out2 && out_map(&m.out2, g.out2, g.n_out, 1, g.num_rows, g.ldo2) != cudaSuccess) st = false;
  m.flags = st ? kBoxStores : 0;
  const long long tiles = (long long)(cdiv(g.num_rows, BM) + g.E) * nN * (g.ksplit > 1 ? g.ksplit : 1);
  if (g.a_mode == ROWS_GATHER) {
    if (g.ksplit > 1) return cudaErrorInvalidValue;
    return swiglu ? launch_g<true, true, true, false, false, false, true>(ta, tb, m, g, nN, tiles, s)
                  : launch_g<true, true, false, false, false, false, true>(ta, tb, m, g, nN, tiles, s);
  }
  if (g.epi != EPI_STORE) return cudaErrorInvalidValue;
  if (g.ksplit > 1) return launch_g<false, true, false, false, true, false, true>(ta, tb, m, g, nN, tiles, s);
  return launch_g<false, true, false, false, false, false, true>(ta, tb, m, g, nN, tiles, s);
}

cudaError_t launch_grouped_gemm_tc(const GroupedGemm& g, cudaStream_t s) {
  if (g.num_rows == 0) return cudaSuccess;
  if (g.E > kMaxE) return cudaErrorInvalidValue;
  if (g.out_f32) return cudaErrorInvalidValue;  // every output of this path is bf16
  if (g.fp8) return launch_grouped_gemm_fp8(g, s);
  if (g.ksplit > 1) {  // split K: the plain-store epilogue of a TMA-fed single-CTA product
    if (g.a_mode != ROWS_GROUPED || g.epi != EPI_STORE || g.partial == nullptr || g.ksplit > cdiv(g.K, BK))
      return cudaErrorInvalidValue;
  }
  const bool swiglu = g.epi == EPI_ACT_FWD && g.act == SMOE_ACT_SWIGLU;
  const int BNo = swiglu ? BN / 2 : BN;
  const int nN = cdiv(g.n_out, BNo);
  const bool gather = g.a_mode == ROWS_GATHER;
  // A gathered product with a short K has little main loop per tile to hide its
  // epilogue behind: half the gather warps become a second epilogue group.  Not for
  // SwiGLU's forward, whose epilogue (half-width tiles) is short and whose gather
  // then sets the pace (measured slower with 4 gather warps).
  const bool shortk = gather && !swiglu && g.K <= kShortK && g.ksplit <= 1;
  // Policy 1 (smoe_set_gemm_policy): long-K products over large expert slices
  // (at least 2048 rows per expert on average, K >= 4096) run TMA-fed ones on CTA
  // pairs (six-stage rings of 32 KB per CTA, half of B per CTA) and gather the
  // others with 4 warps on one CTA.  Either policy walks an expert's tiles in
  // panels of M tiles (map_tile): a wave of 148 CTAs then covers about 16 x 9
  // tiles, whose A rows and weight columns are read by more tiles at once.
  const bool big = g_gemm_policy == 1 && g.ksplit <= 1 && g.K >= 4096 &&
                   (long long)g.num_rows >= 2048LL * g.E;
  const bool pair = big && !gather;
  const bool g128 = big && gather && !shortk;
  CUtensorMap ta, tb;
  cudaError_t e = rows_map(&ta, g.a, g.K, g.a_rows, g.lda, BM);  // unused when gathered
  if (e != cudaSuccess) return e;
  const bool kmaj = g.b_kn == 0;
  // The slab view needs whole 64-column slabs (and SwiGLU's up half to start on one):
  // it never reaches past a row, so every element it addresses is in the tensor.
  // Used for long K only: the Mixtral-shaped down projection (K = 14336) measured 3%
  // faster with it, while the fine-grained sweep's products (K = 512-2048) measured up
  // to 6% slower.  Single CTAs only: CTA pairs (policy 1) keep one load per slab.
  const bool slab = !kmaj && !pair && g.K >= 4096 && g.NW % 64 == 0 && (!swiglu || g.n_out % 64 == 0);
  if (kmaj) {  // W[e] is [NW, K]: dims {K, NW, E}
    const uint64_t dims[3] = {(uint64_t)g.K, (uint64_t)g.NW, (uint64_t)g.E};
    const uint64_t str[2] = {(uint64_t)g.K * 2, (uint64_t)g.NW * g.K * 2};
    // (SwiGLU's forward loads its gate and up rows as two half-height boxes)
    const uint32_t box[3] = {64, (uint32_t)((pair || swiglu) ? BN / 2 : BN), 1};
    e = make_map(&tb, g.b, 3, dims, str, box);
  } else if (slab) {  // W[e] is [K, NW] seen as slabs: dims {64, K, NW / 64, E}
    const uint64_t dims[4] = {64, (uint64_t)g.K, (uint64_t)g.NW / 64, (uint64_t)g.E};
    const uint64_t str[3] = {(uint64_t)g.NW * 2, 128, (uint64_t)g.K * g.NW * 2};
    const uint32_t box[4] = {64, BK, (uint32_t)((pair || swiglu) ? 2 : 4), 1};
    e = make_map(&tb, g.b, 4, dims, str, box);
  } else {  // W[e] is [K, NW]: dims {NW, K, E}
    const uint64_t dims[3] = {(uint64_t)g.NW, (uint64_t)g.K, (uint64_t)g.E};
    const uint64_t str[2] = {(uint64_t)g.NW * 2, (uint64_t)g.K * g.NW * 2};
    const uint32_t box[3] = {64, BK, 1};
    e = make_map(&tb, g.b, 3, dims, str, box);
  }
  if (e != cudaSuccess) return e;
  // Boxed (TMA tensor) epilogue stores when every output is in grouped rows;
  // boxed ACT_BWD input loads when its inputs are in grouped rows.
  EpiMaps m;
  const int parts = (g.act == SMOE_ACT_SWIGLU && g.epi != EPI_STORE) ? 2 : 1;
  bool st = (g.out != nullptr || g.out2 != nullptr) &&
            (g.out == nullptr || g.out_mode == ROWS_GROUPED);
  if (st && g.out && out_map(&m.out, g.out, g.n_out, parts, g.num_rows, g.ldo) != cudaSuccess) st = false;
  if (st && g.out2 && out_map(&m.out2, g.out2, g.n_out, 1, g.num_rows, g.ldo2) != cudaSuccess) st = false;
  const bool need_h = g.out != nullptr && g.act != SMOE_ACT_NONE;
  bool ld = g.epi == EPI_ACT_BWD && g.aux_a_mode == ROWS_GROUPED && !swiglu;
  if (ld && out_map(&m.xa, g.aux_a, g.n_out, 1, g.num_rows, g.ld_aux_a) != cudaSuccess) ld = false;
  if (ld && need_h && out_map(&m.xh, g.aux_h, g.n_out, parts, g.num_rows, g.ld_aux_h) != cudaSuccess) ld = false;
  m.flags = (st ? kBoxStores : 0) | (ld ? kBoxLoads : 0) | (slab ? kSlabB : 0);
  const int tm = pair ? 2 * BM : BM;  // rows per M tile
  // Panels of 16 M tiles (8 on pairs): measured 33% fewer DRAM reads on the
  // Mixtral-shaped down projection and 1.2% less time per step over 20 steps.
  GroupedGemm gp = g;
  gp.panel_m = pair ? 8 : 16;
  const long long tiles = (long long)(cdiv(g.num_rows, tm) + g.E) * nN * (g.ksplit > 1 ? g.ksplit : 1);
  if (g.ksplit > 1) {  // grouped A, plain store (checked above)
    if (kmaj) return launch_g<false, true, false, false, true>(ta, tb, m, gp, nN, tiles, s);
    return launch_g<false, false, false, false, true>(ta, tb, m, gp, nN, tiles, s);
  }
  if (shortk) {
    if (kmaj) return launch_g<true, true, false, false, false, true>(ta, tb, m, gp, nN, tiles, s);
    return launch_g<true, false, false, false, false, true>(ta, tb, m, gp, nN, tiles, s);
  }
#define SMOE_LAUNCH_G(AG, KM, SW)                                                              \
  (pair ? (g128 ? launch_g<AG, KM, SW, true, false, false, false, AG>(ta, tb, m, gp, nN, tiles, s)        \
                : launch_g<AG, KM, SW, true>(ta, tb, m, gp, nN, tiles, s))                               \
        : (g128 ? launch_g<AG, KM, SW, false, false, false, false, AG>(ta, tb, m, gp, nN, tiles, s)       \
                : launch_g<AG, KM, SW, false>(ta, tb, m, gp, nN, tiles, s)))
  if (gather) {
    if (kmaj) return swiglu ? SMOE_LAUNCH_G(true, true, true) : SMOE_LAUNCH_G(true, true, false);
    return swiglu ? SMOE_LAUNCH_G(true, false, true) : SMOE_LAUNCH_G(true, false, false);
  }
  if (kmaj) return swiglu ? SMOE_LAUNCH_G(false, true, true) : SMOE_LAUNCH_G(false, true, false);
  return swiglu ? SMOE_LAUNCH_G(false, false, true) : SMOE_LAUNCH_G(false, false, false);
#undef SMOE_LAUNCH_G
}

cudaError_t launch_dw_gemm_tc(const DwGemm& g_in, cudaStream_t s) {
  if (g_in.E > kMaxE) return cudaErrorInvalidValue;
  // Keep a single gathered operand on the A (128-wide, 16 KB per stage) side:
  // compute dW^T and store it transposed.
  DwGemm g = g_in;
  const bool trans = g_in.b_mode == ROWS_GATHER && g_in.a_mode == ROWS_GROUPED;
  if (trans) {
    g.M = g_in.N; g.N = g_in.M;
    g.a = g_in.b; g.lda = g_in.ldb; g.a_rows = g_in.b_rows; g.a_mode = g_in.b_mode; g.a_fan_out = g_in.b_fan_out;
    g.b = g_in.a; g.ldb = g_in.lda; g.b_rows = g_in.a_rows; g.b_mode = g_in.a_mode; g.b_fan_out = g_in.a_fan_out;
  }
  const int nM = cdiv(g.M, BM), nN = cdiv(g.N, BN);
  const bool ag = g.a_mode == ROWS_GATHER, bg = g.b_mode == ROWS_GATHER;
  // gated rows: the gate multiplies the A operand as it is gathered (a grouped A
  // is then gathered row by row)
  const bool sc = g.row_gates != nullptr;
  // A product with both operands fed by TMA and whole 64-column slabs uses the slab
  // view {64, rows, slabs}: one load per stage and operand instead of one per slab
  // (the view never reaches past a row).  With a gathered operand the gather sets
  // the pace, and the Mixtral-shaped dW measured 1% slower with the slab view.
  const bool pair_b = (sc || (ag && g_gemm_policy == 1 && (long long)g.num_rows >= 2048LL * g.E)) &&
                      !bg && g.M > BM;  // the pair kernel below (half of B per CTA)
  const int slabs = (!ag && !sc && !bg && g.M % 64 == 0 && g.N % 64 == 0) ? 3 : 0;
  CUtensorMap ta, tb;
  cudaError_t e = (slabs & 1) ? slab_map(&ta, g.a, g.M, g.a_rows, g.lda, BK, 2)
                              : rows_map(&ta, g.a, g.M, g.a_rows, g.lda, BK);  // unused when gathered
  if (e != cudaSuccess) return e;
  e = (slabs & 2) ? slab_map(&tb, g.b, g.N, g.b_rows, g.ldb, BK, pair_b ? 2 : 4)
                  : rows_map(&tb, g.b, g.N, g.b_rows, g.ldb, BK);
  if (e != cudaSuccess) return e;
  // fp32 dW as [E, rows, cols] with 32 x 32 boxes: rows = M, cols = N, or the
  // transpose when the kernel computes dW^T
  CUtensorMap td;
  memset(&td, 0, sizeof(td));
  const uint64_t rows = trans ? g.N : g.M, cols = trans ? g.M : g.N;
  const uint64_t ddims[3] = {cols, rows, (uint64_t)g.E};
  const uint64_t dstr[2] = {cols * 4, rows * cols * 4};
  const uint32_t dbox[3] = {32, 32, 1};
  const int d_boxed = make_map(&td, g.dw, 3, ddims, dstr, dbox, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_DATA_TYPE_FLOAT32) == cudaSuccess;
  // Gated rows with B by TMA and at least two 128-column halves of M run on CTA
  // pairs: their six-stage rings keep more gathered stages in flight while the
  // gate pass holds stages back (measured 9% faster than one CTA on the
  // Mixtral-shaped dW2).  Under policy 1 ungated products over large slices (at
  // least 2048 rows per expert on average) do too (2-3% faster on the
  // Mixtral-shaped dW1 and dW2 in short runs below the power cap).
  if (pair_b) {
    const int nMP = cdiv(g.M, 2 * BM);
    const long long ptiles = (long long)g.E * nMP * nN;
    if (!sc)
      return trans ? launch_dp<false, true>(tb, td, d_boxed, slabs, g, nMP, nN, ptiles, s)
                   : launch_dp<false, false>(tb, td, d_boxed, slabs, g, nMP, nN, ptiles, s);
    return trans ? launch_dp<true, true>(tb, td, d_boxed, slabs, g, nMP, nN, ptiles, s)
                 : launch_dp<true, false>(tb, td, d_boxed, slabs, g, nMP, nN, ptiles, s);
  }
  const long long tiles = (long long)g.E * nM * nN;
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
#define SMOE_LAUNCH_D(AG, BG, TR, SC) launch_d<AG, BG, TR, SC>(ta, tb, td, d_boxed, slabs, g, nM, nN, grid, s)
  if (sc) {
    if (bg) return SMOE_LAUNCH_D(true, true, false, true);
    return trans ? SMOE_LAUNCH_D(true, false, true, true) : SMOE_LAUNCH_D(true, false, false, true);
  }
  if (trans) return SMOE_LAUNCH_D(true, false, true, false);
  if (ag) return bg ? SMOE_LAUNCH_D(true, true, false, false) : SMOE_LAUNCH_D(true, false, false, false);
  return SMOE_LAUNCH_D(false, false, false, false);
#undef SMOE_LAUNCH_D
}

}  // namespace smoe

extern "C" int smoe_selftest_wait_timeout(int limit_us, void* stream) {
  using namespace smoe;
  if (limit_us <= 0 || limit_us > 1000000)
    return api_fail(SMOE_ERR_INVALID_ARG, "limit_us must be in (0, 1e6]");
  cudaError_t st;
  unsigned* err = api_error_word(&st);
  if (!err) return api_fail(SMOE_ERR_CUDA, "smoe_selftest_wait_timeout: %s", cudaGetErrorString(st));
  wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(1000ull * (unsigned long long)limit_us, err);
  st = cudaGetLastError();
  return st == cudaSuccess ? SMOE_OK
                           : api_fail(SMOE_ERR_CUDA, "smoe_selftest_wait_timeout: %s", cudaGetErrorString(st));
}
