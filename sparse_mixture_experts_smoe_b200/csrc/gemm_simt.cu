// gemm_simt.cu -- grouped GEMMs of ParallelLinear on the FP32 CUDA cores.
//
// This is the path of the fp32 configuration (tensor cores cannot hold fp32
// operands at fp32 accuracy).  It implements exactly the operations of the
// tcgen05 path in gemm_tc.cu:
//   * grouped-M GEMM: "grouped matrix operations on scattered groups"
//     (tradepoint.io article, method paragraphs): every CTA owns one expert's
//     contiguous slice of the sorted slot list, reads its input rows either
//     grouped or scattered (gathered through sorted_slot, no grouped copy), and
//     writes grouped or scattered rows, with the activation / gate / gate-gradient
//     epilogues fused (library page of arXiv 2403.08245, review 2 summary);
//   * per-expert weight gradient: dW[e] accumulates over the expert's slice in
//     fp32 in ascending row order ("gradients for each expert", same article).
// Tiles: 64 x 64 outputs, 16-deep K steps, 256 threads with 4 x 4 outputs each.
#include "common.cuh"

namespace smoe {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;

template <typename T>
__device__ __forceinline__ float load_b(const T* b, int b_kn, int K, int NW, int e, int k, int n) {
  return b_kn ? to_f(b[((size_t)e * K + k) * NW + n]) : to_f(b[((size_t)e * NW + n) * K + k]);
}

template <typename TO>
__device__ __forceinline__ void store_val(void* out, size_t off, float v) {
  reinterpret_cast<TO*>(out)[off] = from_f<TO>(v);
}

// Find the expert and first row of linear M tile `tile`; false if past the end.
__device__ __forceinline__ bool m_tile_coords(const int32_t* offsets, int E, int tile, int bm,
                                              int& e_out, int& row0, int& row_end) {
  int acc = 0;
  for (int e = 0; e < E; ++e) {
    const int r0 = offsets[e], r1 = offsets[e + 1];
    const int nt = (r1 - r0 + bm - 1) / bm;
    if (tile < acc + nt) {
      e_out = e;
      row0 = r0 + (tile - acc) * bm;
      row_end = r1;
      return true;
    }
    acc += nt;
  }
  return false;
}

template <typename T, int NH>
__global__ void __launch_bounds__(kThreads) grouped_gemm_simt_kernel(GroupedGemm g) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[NH][kBK][kBN + 4];
  __shared__ float red[kBM][kBN / 4 + 1];

  int e, row0, row_end;
  if (!m_tile_coords(g.offsets, g.E, blockIdx.x, kBM, e, row0, row_end)) return;
  const int n0 = blockIdx.y * kBN;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const T* A = reinterpret_cast<const T*>(g.a);
  const T* B = reinterpret_cast<const T*>(g.b);

  float acc[NH][4][4];
#pragma unroll
  for (int h = 0; h < NH; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[h][i][j] = 0.0f;

  for (int k0 = 0; k0 < g.K; k0 += kBK) {
#pragma unroll
    for (int u = 0; u < (kBM * kBK) / kThreads; ++u) {
      const int q = tid + u * kThreads;
      const int r = q / kBK, kk = q % kBK;
      const int i = row0 + r, k = k0 + kk;
      float v = 0.0f;
      if (i < row_end && k < g.K) {
        const int sr = src_row(g.a_mode, i, g.sorted_slot, g.a_fan_out);
        v = to_f(A[(size_t)sr * g.lda + k]);
      }
      As[kk][r] = v;
    }
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int u = 0; u < (kBN * kBK) / kThreads; ++u) {
        const int q = tid + u * kThreads;
        // coalesce along the contiguous dimension of W
        const int n = g.b_kn ? q % kBN : q / kBK;
        const int kk = g.b_kn ? q / kBN : q % kBK;
        const int c = n0 + n, k = k0 + kk;
        float v = 0.0f;
        if (c < g.n_out && k < g.K) v = load_b(B, g.b_kn, g.K, g.NW, e, k, c + h * g.n_out);
        Bs[h][kk][n] = v;
      }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[NH][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j) b[h][j] = Bs[h][kk][tx * 4 + j];
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[h][i][j] = fmaf(a[i], b[h][j], acc[h][i][j]);
    }
    __syncthreads();
  }

  // ---- epilogue ----
  const T* AUXA = reinterpret_cast<const T*>(g.aux_a);
  const T* AUXH = reinterpret_cast<const T*>(g.aux_h);
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const int r = ty * 4 + ii;
    const int i = row0 + r;
    const bool row_ok = i < row_end;
    const int p = row_ok ? g.sorted_slot[i] : 0;
    const int orow = g.out_mode == ROWS_GROUPED ? i : p;
    const float gate = (row_ok && g.gates) ? g.gates[p] : 1.0f;
    float dg_part = 0.0f;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int c = n0 + tx * 4 + jj;
      if (!row_ok || c >= g.n_out) continue;
      const float v = acc[0][ii][jj];
      if (g.epi == EPI_STORE) {
        const size_t off = (size_t)orow * g.ldo + c;
        if (g.out_f32) store_val<float>(g.out, off, gate * v); else store_val<T>(g.out, off, gate * v);
      } else if (g.epi == EPI_ACT_FWD) {
        if (NH == 2) {
          const float u = acc[NH - 1][ii][jj];
          store_val<T>(g.out, (size_t)orow * g.ldo + c, v);
          store_val<T>(g.out, (size_t)orow * g.ldo + g.n_out + c, u);
          store_val<T>(g.out2, (size_t)orow * g.ldo2 + c, silu_f(v) * u);
        } else {
          store_val<T>(g.out, (size_t)orow * g.ldo + c, v);
          store_val<T>(g.out2, (size_t)orow * g.ldo2 + c, gelu_tanh_f(v));
        }
      } else {  // EPI_ACT_BWD: v = dA'
        const int ar = src_row(g.aux_a_mode, i, g.sorted_slot, g.aux_a_fan_out);
        const float av = to_f(AUXA[(size_t)ar * g.ld_aux_a + c]);
        dg_part = fmaf(v, av, dg_part);
        if (g.out2) store_val<T>(g.out2, (size_t)i * g.ldo2 + c, gate * av);
        const float da = gate * v;
        if (g.act == SMOE_ACT_SWIGLU) {
          const float hg = to_f(AUXH[(size_t)i * g.ld_aux_h + c]);
          const float hu = to_f(AUXH[(size_t)i * g.ld_aux_h + g.n_out + c]);
          const size_t o = (size_t)orow * g.ldo;
          const float d_g = da * hu * silu_grad_f(hg), d_u = da * silu_f(hg);
          if (g.out_f32) { store_val<float>(g.out, o + c, d_g); store_val<float>(g.out, o + g.n_out + c, d_u); }
          else { store_val<T>(g.out, o + c, d_g); store_val<T>(g.out, o + g.n_out + c, d_u); }
        } else {
          float dh = da;
          if (g.act == SMOE_ACT_GELU_TANH) dh *= gelu_tanh_grad_f(to_f(AUXH[(size_t)i * g.ld_aux_h + c]));
          const size_t o = (size_t)orow * g.ldo + c;
          if (g.out_f32) store_val<float>(g.out, o, dh); else store_val<T>(g.out, o, dh);
        }
      }
    }
    if (g.epi == EPI_ACT_BWD) red[r][tx] = dg_part;
  }
  if (g.epi == EPI_ACT_BWD) {
    __syncthreads();
    if (tid < kBM) {
      const int i = row0 + tid;
      if (i < row_end) {
        float s = 0.0f;
        for (int q = 0; q < kBN / 4; ++q) s += red[tid][q];
        g.dg_partial[(size_t)i * g.dg_ld + blockIdx.y] = s;
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) dw_gemm_simt_kernel(DwGemm g) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  const int e = blockIdx.z;
  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const T* A = reinterpret_cast<const T*>(g.a);
  const T* B = reinterpret_cast<const T*>(g.b);
  const int r_begin = g.offsets[e], r_end = g.offsets[e + 1];
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  for (int r0 = r_begin; r0 < r_end; r0 += kBK) {
#pragma unroll
    for (int u = 0; u < (kBM * kBK) / kThreads; ++u) {
      const int q = tid + u * kThreads;
      const int kk = q / kBM, m = q % kBM;
      const int r = r0 + kk;
      float va = 0.0f, vb = 0.0f;
      if (r < r_end) {
        if (m0 + m < g.M) {
          va = to_f(A[(size_t)src_row(g.a_mode, r, g.sorted_slot, g.a_fan_out) * g.lda + m0 + m]);
          if (g.row_gates) va *= g.row_gates[g.sorted_slot[r]];
        }
        if (n0 + m < g.N) vb = to_f(B[(size_t)src_row(g.b_mode, r, g.sorted_slot, g.b_fan_out) * g.ldb + n0 + m]);
      }
      As[kk][m] = va;
      Bs[kk][m] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < g.M && n < g.N) g.dw[((size_t)e * g.M + m) * g.N + n] = acc[i][j];
    }
}

template <typename T>
cudaError_t launch_grouped_t(const GroupedGemm& g, cudaStream_t s) {
  const int m_tiles = cdiv(g.num_rows, kBM) + g.E;  // upper bound; extra CTAs exit
  dim3 grid(m_tiles, cdiv(g.n_out, kBN));
  const bool swiglu_fwd = g.epi == EPI_ACT_FWD && g.act == SMOE_ACT_SWIGLU;
  if (swiglu_fwd) grouped_gemm_simt_kernel<T, 2><<<grid, kThreads, 0, s>>>(g);
  else grouped_gemm_simt_kernel<T, 1><<<grid, kThreads, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace

int simt_tile_cols() { return kBN; }

cudaError_t launch_grouped_gemm_simt(const GroupedGemm& g, smoe_dtype dt, cudaStream_t s) {
  if (g.num_rows == 0) return cudaSuccess;
  return dt == SMOE_BF16 ? launch_grouped_t<bf16>(g, s) : launch_grouped_t<float>(g, s);
}

cudaError_t launch_dw_gemm_simt(const DwGemm& g, smoe_dtype dt, cudaStream_t s) {
  dim3 grid(cdiv(g.M, kBM), cdiv(g.N, kBN), g.E);
  if (dt == SMOE_BF16) dw_gemm_simt_kernel<bf16><<<grid, kThreads, 0, s>>>(g);
  else dw_gemm_simt_kernel<float><<<grid, kThreads, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace smoe
