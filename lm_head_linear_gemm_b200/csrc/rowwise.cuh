// Row-wise kernels around the tensor-core contractions: target preparation, the
// cross-slab log-sum-exp merge with the gradient-operand patch, the loss reduction
// and the upstream-gradient scaling.  All reductions run in a fixed order, so
// results are bitwise reproducible.
#pragma once
#include <cuda_fp8.h>

#include "sm100.cuh"

namespace flce {

struct DevHeader {
  uint32_t status;           // DEV_* bits
  uint32_t pad0;
  long long n_valid;         // rows whose target enters the loss
  uint32_t reserved[60];
};
static_assert(sizeof(DevHeader) == 256, "header is one 256-byte block");

// One block: effective targets (t, or -1 when ignored or invalid), count of rows in
// the loss, and the bad-target bit.  Resets the status word for this call.
__global__ void __launch_bounds__(1024) prep_targets_kernel(const long long* __restrict__ targets,
                                                            long long N, long long Vreal,
                                                            long long ignore_index,
                                                            int* __restrict__ tgt,
                                                            DevHeader* __restrict__ hdr) {
  __shared__ int s_count[32];
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  int count = 0, bad = 0;
  for (long long i = threadIdx.x; i < N; i += blockDim.x) {
    const long long t = targets[i];
    const bool ignored = t == ignore_index;
    const bool in_range = t >= 0 && t < Vreal;
    const bool ok = in_range && !ignored;
    count += ok ? 1 : 0;
    bad |= (!ok && !ignored) ? 1 : 0;
    tgt[i] = ok ? static_cast<int>(t) : -1;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) count += __shfl_xor_sync(0xffffffffu, count, o);
  if ((threadIdx.x & 31) == 0) s_count[threadIdx.x >> 5] = count;
  if (bad) atomicOr(&s_bad, 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    long long total = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) total += s_count[w];
    hdr->n_valid = total;
    hdr->status = s_bad ? DEV_BAD_TARGET : 0u;
  }
}

// Per chunk of Nc rows (one block each): effective targets, and the compaction of the rows in the
// loss that the gradient contractions run over.  pos[i] is row i's position among its chunk's
// rows in the loss (-1 when ignored or invalid), orig[c*Nc + q] the chunk-local index of the
// chunk's q-th row in the loss, cnt[c] their number and bad[c] whether the chunk holds a target
// outside [0, Vreal) that is not ignore_index.  Rows keep their order (a stable partition).
__global__ void __launch_bounds__(1024) prep_chunks_kernel(const long long* __restrict__ targets,
                                                           long long N, long long Nc,
                                                           long long Vreal, long long ignore_index,
                                                           int* __restrict__ tgt,
                                                           int* __restrict__ pos,
                                                           int* __restrict__ orig,
                                                           int* __restrict__ cnt,
                                                           int* __restrict__ bad) {
  __shared__ int s_scan[32];
  __shared__ int s_base;
  __shared__ int s_bad;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const long long c0 = static_cast<long long>(blockIdx.x) * Nc;
  const long long c1 = c0 + Nc < N ? c0 + Nc : N;
  if (threadIdx.x == 0) {
    s_base = 0;
    s_bad = 0;
  }
  __syncthreads();
  for (long long b = c0; b < c1; b += blockDim.x) {
    const long long i = b + threadIdx.x;
    int ok = 0;
    if (i < c1) {
      const long long t = targets[i];
      const bool ignored = t == ignore_index;
      ok = (t >= 0 && t < Vreal && !ignored) ? 1 : 0;
      if (!ok && !ignored) s_bad = 1;
      tgt[i] = ok ? static_cast<int>(t) : -1;
    }
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) s_scan[w] = __popc(m);
    __syncthreads();
    if (w == 0) {
      int v = lane < nw ? s_scan[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      s_scan[lane] = v;                                  // inclusive over warps
    }
    __syncthreads();
    const int base = s_base;
    const int total = s_scan[nw - 1];
    const int p = base + (w > 0 ? s_scan[w - 1] : 0) + __popc(m & ((1u << lane) - 1u));
    if (i < c1) {
      pos[i] = ok ? p : -1;
      if (ok) orig[c0 + p] = static_cast<int>(i - c0);
    }
    __syncthreads();
    if (threadIdx.x == 0) s_base = base + total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    cnt[blockIdx.x] = s_base;
    bad[blockIdx.x] = s_bad;
  }
}

// One block: rows in the loss and the bad-target bit over all chunks (fixed order).  Resets the
// status word for this call.
__global__ void __launch_bounds__(256) prep_total_kernel(const int* __restrict__ cnt,
                                                         const int* __restrict__ bad, int n_chunks,
                                                         DevHeader* __restrict__ hdr) {
  __shared__ long long s_n[256];
  __shared__ int s_b[256];
  long long n = 0;
  int b = 0;
  for (int c = threadIdx.x; c < n_chunks; c += blockDim.x) {
    n += cnt[c];
    b |= bad[c];
  }
  s_n[threadIdx.x] = n;
  s_b[threadIdx.x] = b;
  __syncthreads();
  for (int k = blockDim.x >> 1; k > 0; k >>= 1) {
    if (static_cast<int>(threadIdx.x) < k) {
      s_n[threadIdx.x] += s_n[threadIdx.x + k];
      s_b[threadIdx.x] |= s_b[threadIdx.x + k];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    hdr->n_valid = s_n[0];
    hdr->status = s_b[0] ? DEV_BAD_TARGET : 0u;
  }
}

struct RowFinishParams {
  int rows;                     // rows of this pass
  int d, Vpad;
  int a_ld;                     // row stride of A (elements, >= Vpad)
  int n_slabs;
  float cap;                    // softcap value (the exp reference when fixed_ref)
  int fixed_ref;                // 1: partials are sum-exp against cap; 0: (max, sum-exp) pairs
  int from_partials;            // 1: lse from the per-slab partials; 0: lse given (lse_in)
  int want_grads;               // 1: also r, the target patch of A and Xs = r . X
  const float* partial;         // [rows][n_slabs] (x2 when cap <= 0)
  const int* tgt;               // [rows]
  const float* s_t;             // [rows]
  const float* der_t;           // [rows]
  const float* e_t;             // [rows]
  const float* lse_in;          // [rows] (from_partials == 0)
  float* lse_out;               // [rows] (from_partials == 1)
  float* row_loss;              // [rows] lse - s_t for rows in the loss, else 0 (from_partials)
  const DevHeader* hdr;         // n_valid
  const long long* nv_total;    // rows in the loss over all data-parallel ranks, or null (= local)
  const float* grad_out;        // device scalar g, or null for g = 1
  float* r;                     // [rows]
  __nv_bfloat16* A;             // [rows][Vpad]
  const __nv_bfloat16* X;       // [rows][d]
  __nv_bfloat16* Xs;            // [rows][d]
  // Compaction (want_grads with pos != null): r, Xs and the rows of A are indexed by the row's
  // position among the chunk's rows in the loss; rows not in the loss get a zero dX row here
  // (the dX contraction skips them), and `ktail` extra warps zero the rows [cnt, cnt rounded up
  // to ktail) of A and Xs, ktail being the dW contraction's k-block (64 rows for bf16, 128 for
  // 8-bit operands), so that its last k-block adds nothing.
  const int* pos;               // [rows] position or -1
  const int* cnt;               // this chunk's number of rows in the loss
  int ktail;                    // rows per k-block of the dW contraction (64 or 128)
  __nv_bfloat16* dX;            // [rows][d] this chunk's dX rows
  // 8-bit gradient operands (fp8 = 1, with compaction and the fixed reference): the row's
  // softmax gradient normalised by S and scaled by 2^15, q_j = e5m2(A'_j / S * 2^15), replaces
  // the bf16 row of A in place (its first Vpad bytes; rows keep their 2 Vpad-byte stride), and
  // the row's e4m3 X8 bytes are copied to Xs8 at its compacted position.
  int fp8;
  const uint8_t* X8;            // [rows][d] this chunk's e4m3 rows
  uint8_t* Xs8;                 // [rows][d]
  // The final RMSNorm's backward folded into dX (fixed reference, from partials): the row term
  // c_i = mean_k x_ik dX_ik = (1/d) sum_j dz_ij z_ij = r_i (Q_i - S_i der_t z_t) / d, Q_i the
  // sum of the per-slab partials of A_ij z_ij (A before the target patch); 0 outside the loss.
  const float* q_partial;       // [rows][n_slabs], or null (no fold)
  const float* z_t;             // [rows] target logit before the softcap
  float* cdot;                  // [rows] c_i (indexed like r)
};

__device__ __forceinline__ void zero_row_bf16(__nv_bfloat16* row, int n, int lane) {
  for (int k = lane * 8; k < n; k += 256) *reinterpret_cast<uint4*>(row + k) = make_uint4(0, 0, 0, 0);
}

// One warp: the e5m2 gradient row of a row in the loss (see RowFinishParams::fp8), written over
// the first half of the bf16 row it is formed from.  The row is converted in batches: each batch
// reads its bf16 elements into registers, the warp synchronises, then writes their codes, which
// land on bytes whose bf16 values this or an earlier batch has already read.
template <class P>
__device__ __forceinline__ void encode_row_e5m2(const P& p, int row, int at, int t, float S) {
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* arow = p.A + static_cast<size_t>(at) * p.a_ld;
  uint8_t* qrow = reinterpret_cast<uint8_t*>(p.A + static_cast<size_t>(at) * p.a_ld);
  // the target element as the bf16 path stores it, (1 - tanh^2)(e_t - S) rounded to bf16
  const float pv = __bfloat162float(__float2bfloat16_rn(p.der_t[row] * (p.e_t[row] - S)));
  const float f = 32768.0f / S;
  constexpr int B = 4;                                 // groups of 8 elements per lane per batch
  for (int base = 0; base < p.Vpad; base += 32 * 8 * B) {
    uint4 v[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int k = base + (b * 32 + lane) * 8;
      if (k < p.Vpad) v[b] = *reinterpret_cast<const uint4*>(arow + k);
    }
    __syncwarp();
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int k = base + (b * 32 + lane) * 8;
      if (k < p.Vpad) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[b]);
        float x[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f2 = __bfloat1622float2(h[q]);
          x[2 * q] = f2.x;
          x[2 * q + 1] = f2.y;
        }
        if (static_cast<unsigned>(t - k) < 8u) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q == t - k) x[q] = pv;
        }
        uint32_t w[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * q] * f, x[4 * q + 1] * f),
                                                       __NV_SATFINITE, __NV_E5M2);
          const uint32_t hi = __nv_cvt_float2_to_fp8x2(
              make_float2(x[4 * q + 2] * f, x[4 * q + 3] * f), __NV_SATFINITE, __NV_E5M2);
          w[q] = lo | (hi << 16);
        }
        *reinterpret_cast<uint2*>(qrow + k) = make_uint2(w[0], w[1]);
      }
    }
    __syncwarp();
  }
  const uint8_t* xr = p.X8 + static_cast<size_t>(row) * p.d;
  uint8_t* xs = p.Xs8 + static_cast<size_t>(at) * p.d;
  for (int k = lane * 16; k < p.d; k += 512)
    *reinterpret_cast<uint4*>(xs + k) = *reinterpret_cast<const uint4*>(xr + k);
}

// One warp per row (plus, when compacting, 64 warps that clear the tail rows).
__global__ void __launch_bounds__(256) row_finish_kernel(const RowFinishParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= p.rows) {
    if (p.want_grads && p.pos != nullptr && warp < p.rows + p.ktail) {
      const int m = *p.cnt;
      const int q = m + (warp - p.rows);
      if (q < (m + p.ktail - 1) / p.ktail * p.ktail && q < p.rows) {
        zero_row_bf16(p.A + static_cast<size_t>(q) * p.a_ld, p.Vpad, lane);
        if (p.fp8)
          zero_row_bf16(reinterpret_cast<__nv_bfloat16*>(p.Xs8 + static_cast<size_t>(q) * p.d),
                        p.d / 2, lane);
        else
          zero_row_bf16(p.Xs + static_cast<size_t>(q) * p.d, p.d, lane);
      }
    }
    return;
  }
  const int row = warp;
  float lse, S = 1.f, ref;
  if (p.from_partials) {
    if (p.fixed_ref) {
      const float* pp = p.partial + static_cast<size_t>(row) * p.n_slabs;
      float acc = 0.f;
      for (int k = lane; k < p.n_slabs; k += 32) acc += pp[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      S = acc;
      ref = p.cap;
      lse = ref + logf(S);
    } else {
      const float* pp = p.partial + static_cast<size_t>(row) * p.n_slabs * 2;
      float m = -INFINITY;
      for (int k = lane; k < p.n_slabs; k += 32) m = fmaxf(m, pp[2 * k]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float l = 0.f;
      for (int k = lane; k < p.n_slabs; k += 32) {
        const float mk = pp[2 * k];
        if (mk != -INFINITY) l += pp[2 * k + 1] * expf(mk - m);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      lse = m + logf(l);
      ref = lse;
      S = 1.f;
    }
  } else {
    lse = p.lse_in[row];
    ref = p.fixed_ref ? p.cap : lse;
    S = p.fixed_ref ? expf(lse - ref) : 1.f;
  }
  float Q = 0.f;                                  // RMSNorm fold: sum_j A_ij z_ij
  if (p.q_partial != nullptr) {
    const float* qp = p.q_partial + static_cast<size_t>(row) * p.n_slabs;
    for (int k = lane; k < p.n_slabs; k += 32) Q += qp[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Q += __shfl_xor_sync(0xffffffffu, Q, o);
  }
  const int t = p.tgt[row];
  const bool valid = t >= 0;
  if (lane == 0 && p.from_partials) {
    p.lse_out[row] = lse;
    p.row_loss[row] = valid ? lse - p.s_t[row] : 0.f;
  }
  if (!p.want_grads) return;
  const long long nv = p.nv_total != nullptr ? *p.nv_total : p.hdr->n_valid;
  const float g = p.grad_out ? *p.grad_out : 1.f;
  const float r = (valid && nv > 0) ? g / (static_cast<float>(nv) * S) : 0.f;
  int at = row;                                   // row of r, A and Xs
  if (p.pos != nullptr) {
    if (!valid) {                                 // not in the loss: dX row is zero
      zero_row_bf16(p.dX + static_cast<size_t>(row) * p.d, p.d, lane);
      return;
    }
    at = p.pos[row];
  }
  if (p.fp8) {
    encode_row_e5m2(p, row, at, t, S);
    return;
  }
  if (p.cdot != nullptr && lane == 0)
    p.cdot[at] = r != 0.f ? r * (Q - S * p.der_t[row] * p.z_t[row]) / static_cast<float>(p.d)
                          : 0.f;
  if (lane == 0) {
    p.r[at] = r;
    if (valid) {
      const float patched = p.der_t[row] * (p.e_t[row] - S);
      p.A[static_cast<size_t>(at) * p.a_ld + t] = __float2bfloat16_rn(patched);
    }
  }
  const __nv_bfloat16* xr = p.X + static_cast<size_t>(row) * p.d;
  __nv_bfloat16* xs = p.Xs + static_cast<size_t>(at) * p.d;
  for (int k = lane * 8; k < p.d; k += 256) {
    const uint4 raw = *reinterpret_cast<const uint4*>(xr + k);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint4 w;
    uint32_t* wo = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(h[q]);
      wo[q] = pack_bf16x2(f.x * r, f.y * r);
    }
    *reinterpret_cast<uint4*>(xs + k) = w;
  }
}

// One block: loss = sum(row_loss) / n_valid, 0 when no row is in the loss.  With nv_total (the
// count over all data-parallel ranks) the result is this rank's share of the global mean.
__global__ void __launch_bounds__(1024) loss_kernel(const float* __restrict__ row_loss, long long N,
                                                    const DevHeader* __restrict__ hdr,
                                                    const long long* __restrict__ nv_total,
                                                    float* __restrict__ loss) {
  __shared__ double s_part[1024];
  double acc = 0.0;
  for (long long i = threadIdx.x; i < N; i += blockDim.x) acc += static_cast<double>(row_loss[i]);
  s_part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) s_part[threadIdx.x] += s_part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const long long nv = nv_total != nullptr ? *nv_total : hdr->n_valid;
    loss[0] = nv > 0 ? static_cast<float>(s_part[0] / static_cast<double>(nv)) : 0.f;
  }
}

// dX *= g, dW *= g (and dg *= g, fp32) for gradients formed with g = 1; returns at once when
// g == 1.  dW is fp32
// (nW = elements / 4, float4 groups) or bf16 (dW_bf16 = 1, nW = elements / 8, groups of 8).
__global__ void scale_grads_kernel(__nv_bfloat16* __restrict__ dX, long long nX8,
                                   void* __restrict__ dW, long long nW, int dW_bf16,
                                   const float* __restrict__ grad_out,
                                   float* __restrict__ dg = nullptr, long long n_dg = 0) {
  const float g = *grad_out;
  if (g == 1.f) return;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  auto scale_bf16x8 = [g](uint4* p) {
    uint4 raw = *p;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(h[q]);
      h[q] = __floats2bfloat162_rn(f.x * g, f.y * g);
    }
    *p = raw;
  };
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < nX8;
       i += stride)
    scale_bf16x8(reinterpret_cast<uint4*>(dX) + i);
  if (dW != nullptr) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < nW;
         i += stride) {
      if (dW_bf16) {
        scale_bf16x8(reinterpret_cast<uint4*>(dW) + i);
      } else {
        float4 v = reinterpret_cast<float4*>(dW)[i];
        v.x *= g;
        v.y *= g;
        v.z *= g;
        v.w *= g;
        reinterpret_cast<float4*>(dW)[i] = v;
      }
    }
  }
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_dg;
       i += stride)
    dg[i] *= g;
}

// ---------------------------------------------------------------- tensorwise e4m3 quantisation
// scale = amax(|x|) / 448 (448 = largest finite e4m3), q = e4m3(x / scale) rounded to nearest
// even and saturated to the finite range.  The amax is kept as the bit pattern of a
// non-negative float in the scale slot (bit order = value order), then turned into the scale.
__global__ void zero_u32_kernel(uint32_t* p) { *p = 0u; }

__global__ void amax_bf16_kernel(const __nv_bfloat16* __restrict__ x, long long n,
                                 uint32_t* __restrict__ amax_bits) {
  float m = 0.f;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += stride)
    m = fmaxf(m, fabsf(__bfloat162float(x[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__global__ void quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x, long long n,
                                     uint8_t* __restrict__ q, const uint32_t* __restrict__ amax_bits) {
  const float amax = __uint_as_float(*amax_bits);
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += stride)
    q[i] = static_cast<uint8_t>(
        __nv_cvt_float_to_fp8(__fdiv_rn(__bfloat162float(x[i]), scale), __NV_SATFINITE, __NV_E4M3));
}

__global__ void finish_scale_kernel(uint32_t* amax_bits) {
  const float amax = __uint_as_float(*amax_bits);
  *reinterpret_cast<float*>(amax_bits) = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// One block: number of rows whose target enters the loss (t != ignore_index, 0 <= t < Vreal).
__global__ void __launch_bounds__(1024) count_valid_kernel(const long long* __restrict__ targets,
                                                           long long N, long long Vreal,
                                                           long long ignore_index,
                                                           long long* __restrict__ out) {
  __shared__ long long s_count[32];
  long long count = 0;
  for (long long i = threadIdx.x; i < N; i += blockDim.x) {
    const long long t = targets[i];
    count += (t != ignore_index && t >= 0 && t < Vreal) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) count += __shfl_xor_sync(0xffffffffu, count, o);
  if ((threadIdx.x & 31) == 0) s_count[threadIdx.x >> 5] = count;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long total = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) total += s_count[w];
    *out = total;
  }
}

// ---------------------------------------------------------------- final RMSNorm before the head
// x_i = h_i * rstd_i * gamma, rstd_i = 1 / sqrt(mean_k h_ik^2 + eps); fp32 arithmetic, bf16 x.
// One warp per row; every lane handles 8 contiguous columns per step (d % 8 == 0).
__global__ void __launch_bounds__(256) rmsnorm_fwd_kernel(const __nv_bfloat16* __restrict__ H,
                                                          const __nv_bfloat16* __restrict__ gamma,
                                                          float eps, long long N, int d,
                                                          __nv_bfloat16* __restrict__ X,
                                                          float* __restrict__ rstd_out) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const __nv_bfloat16* h = H + row * d;
  float ss = 0.f;
  for (int k = lane * 8; k < d; k += 256) {
    const uint4 raw = *reinterpret_cast<const uint4*>(h + k);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(p2[q]);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rstd = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
  if (lane == 0) rstd_out[row] = rstd;
  __nv_bfloat16* x = X + row * d;
  for (int k = lane * 8; k < d; k += 256) {
    const uint4 raw = *reinterpret_cast<const uint4*>(h + k);
    const uint4 graw = *reinterpret_cast<const uint4*>(gamma + k);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&graw);
    uint4 w;
    uint32_t* wo = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(p2[q]);
      const float2 g = __bfloat1622float2(g2[q]);
      wo[q] = pack_bf16x2(f.x * rstd * g.x, f.y * rstd * g.y);
    }
    *reinterpret_cast<uint4*>(x + k) = w;
  }
}

// dH_i = rstd_i (g_i - xh_i mean_k(g_ik xh_ik)) with xh = h * rstd and g = dX * gamma.
__global__ void __launch_bounds__(256) rmsnorm_bwd_rows_kernel(
    const __nv_bfloat16* __restrict__ H, const __nv_bfloat16* __restrict__ gamma,
    const float* __restrict__ rstd_in, const __nv_bfloat16* __restrict__ dX, long long N, int d,
    __nv_bfloat16* __restrict__ dH) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const float rstd = rstd_in[row];
  const __nv_bfloat16* h = H + row * d;
  const __nv_bfloat16* dx = dX + row * d;
  float dot = 0.f;
  for (int k = lane * 8; k < d; k += 256) {
    const uint4 hr = *reinterpret_cast<const uint4*>(h + k);
    const uint4 dr = *reinterpret_cast<const uint4*>(dx + k);
    const uint4 gr = *reinterpret_cast<const uint4*>(gamma + k);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hr);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dr);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gr);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 hf = __bfloat1622float2(h2[q]);
      const float2 df = __bfloat1622float2(d2[q]);
      const float2 gf = __bfloat1622float2(g2[q]);
      dot = fmaf(df.x * gf.x, hf.x * rstd, dot);
      dot = fmaf(df.y * gf.y, hf.y * rstd, dot);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  const float mean_dot = dot / static_cast<float>(d);
  __nv_bfloat16* out = dH + row * d;
  for (int k = lane * 8; k < d; k += 256) {
    const uint4 hr = *reinterpret_cast<const uint4*>(h + k);
    const uint4 dr = *reinterpret_cast<const uint4*>(dx + k);
    const uint4 gr = *reinterpret_cast<const uint4*>(gamma + k);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hr);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dr);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gr);
    uint4 w;
    uint32_t* wo = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 hf = __bfloat1622float2(h2[q]);
      const float2 df = __bfloat1622float2(d2[q]);
      const float2 gf = __bfloat1622float2(g2[q]);
      wo[q] = pack_bf16x2(rstd * (df.x * gf.x - hf.x * rstd * mean_dot),
                          rstd * (df.y * gf.y - hf.y * rstd * mean_dot));
    }
    *reinterpret_cast<uint4*>(out + k) = w;
  }
}

// dgamma_k = sum_i dX_ik h_ik rstd_i in two deterministic stages: per block of `rows_per_part`
// rows a partial sum per column, then the partials summed in order.  Each thread owns two
// adjacent columns, so a warp reads whole 128-byte lines of each row.
__global__ void __launch_bounds__(256) rmsnorm_dgamma_partial_kernel(
    const __nv_bfloat16* __restrict__ H, const float* __restrict__ rstd_in,
    const __nv_bfloat16* __restrict__ dX, long long N, int d, int rows_per_part,
    float* __restrict__ partial) {
  const int k = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (k >= d) return;
  const long long r0 = static_cast<long long>(blockIdx.y) * rows_per_part;
  const long long r1 = r0 + rows_per_part < N ? r0 + rows_per_part : N;
  float acc0 = 0.f, acc1 = 0.f;
  for (long long i = r0; i < r1; ++i) {
    const float2 h = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(H + i * d + k));
    const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dX + i * d + k));
    const float r = rstd_in[i];
    acc0 = fmaf(g.x, h.x * r, acc0);
    acc1 = fmaf(g.y, h.y * r, acc1);
  }
  float* prow = partial + static_cast<long long>(blockIdx.y) * d;
  prow[k] = acc0;
  prow[k + 1] = acc1;
}

// dgamma (+)= the column sums of one chunk's dX . xh, from the dX epilogue's per-32-row-block
// partials over the blocks of the chunk's rows (its rows in the loss when compacted: a device-side
// count).  A block of 32 x 8 threads takes 32 columns: thread row y sums the blocks b = y mod 8
// in order, then the eight sums are added in order (deterministic).
__global__ void __launch_bounds__(256) rmsnorm_dgamma_chunk_kernel(
    const float* __restrict__ partial, int d, int rows, const int* __restrict__ cnt,
    float* __restrict__ dgamma, int accumulate) {
  __shared__ float part[8][32];
  const int k = blockIdx.x * 32 + threadIdx.x;
  const int m = cnt != nullptr ? *cnt : rows;
  const int blocks = (m + 31) / 32;
  float acc = 0.f;
  if (k < d)
    for (int b = threadIdx.y; b < blocks; b += 8) acc += partial[static_cast<long long>(b) * d + k];
  part[threadIdx.y][threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.y == 0 && k < d) {
    float sum = 0.f;
#pragma unroll
    for (int y = 0; y < 8; ++y) sum += part[y][threadIdx.x];
    dgamma[k] = accumulate ? dgamma[k] + sum : sum;
  }
}

__global__ void rmsnorm_dgamma_final_kernel(const float* __restrict__ partial, int parts, int d,
                                            float* __restrict__ dgamma, int accumulate) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= d) return;
  float acc = 0.f;
  for (int b = 0; b < parts; ++b) acc += partial[static_cast<long long>(b) * d + k];
  dgamma[k] = accumulate ? dgamma[k] + acc : acc;
}

// Self-test of the bounded wait used by every pipeline barrier: one thread initialises an
// mbarrier that expects one arrival, never arrives, and waits on it with the given limit.  The
// wait gives up, raises DEV_TIMEOUT in *status and the kernel returns normally.
__global__ void wait_timeout_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  mbar_wait_bounded(&bar, 0, status, limit_ns);
}

// Factors of the 8-bit gradient contractions: the e5m2 codes carry dz * Nv/g * 2^15, the e4m3
// operands W8 and X8 their tensorwise scales, so dX = [g/(Nv 2^15) sW] (q W8) and
// dW = [g/(Nv 2^15) sX] (q^T Xs8).  out = {dX factor, dW factor}; 0 when no row is in the loss.
__global__ void fp8_grad_scales_kernel(const DevHeader* __restrict__ hdr,
                                       const long long* __restrict__ nv_total,
                                       const float* __restrict__ grad_scale,
                                       const float* __restrict__ scale_w,
                                       const float* __restrict__ scale_x, float* __restrict__ out) {
  const long long nv = nv_total != nullptr ? *nv_total : hdr->n_valid;
  const float g = grad_scale != nullptr ? *grad_scale : 1.f;
  const float base = nv > 0 ? g / (static_cast<float>(nv) * 32768.0f) : 0.f;
  out[0] = base * *scale_w;
  out[1] = base * *scale_x;
}

// Writes loss = 0 (used for N = 0, where nothing else runs).
__global__ void zero_loss_kernel(float* loss) { loss[0] = 0.f; }

}  // namespace flce
