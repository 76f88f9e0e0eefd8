// Weight-oscillation tracker (sm_100a) and the synthetic update that drives
// it.
//
// Source: "ALTO MXFP4 training — Weight de-oscillation — What does it mean?":
// over a window of P optimizer steps, accumulate per element how far the
// master weight travelled (d_w) and how far its quantized value jumped (d_Q);
// at the window end flag d_Q / d_w > threshold and snap flagged weights to
// the centre of their current bin. The extra state is the two distances and
// a weight snapshot; no matrix multiplies are added.
//
// Per step and element: d_w += |w - w_snap|, d_q += |DQ(w) - DQ(w_snap)|
// (DQ = 1x32 RNE quantize-dequantize, values exact in fp32), w_snap = w;
// all fp32 with explicit round-to-nearest intrinsics, so no multiply-add is
// ever fused. The flag test d_q > threshold * d_w never divides, so 0/0 is
// never flagged and a weight that did not move but whose bin changed (its
// group scale moved) is. Four threads share a 1x32 group of all four arrays
// (8 elements each, 2 x 16-byte loads per array), both group maxima come
// from quad shuffles. 28 bytes per element move per step.
#include "launch.cuh"
#include "mxfp4_device.cuh"

namespace mxfp4 {

namespace {

constexpr int kOscThreads = 256;

__device__ __forceinline__ void load8(const float* p, float* v) {
  const uint4 a = ld_l1(p), b = ld_l1(p + 4);
  v[0] = __uint_as_float(a.x), v[1] = __uint_as_float(a.y);
  v[2] = __uint_as_float(a.z), v[3] = __uint_as_float(a.w);
  v[4] = __uint_as_float(b.x), v[5] = __uint_as_float(b.y);
  v[6] = __uint_as_float(b.z), v[7] = __uint_as_float(b.w);
}

__device__ __forceinline__ void store8(float* p, const float* v) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

// 1x32 RNE quantize-dequantize of this thread's 8 elements of a group.
__device__ __forceinline__ void dq8(const float* w, float* q) {
  uint32_t amax = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) amax = max(amax, __float_as_uint(w[j]) & 0x7FFFFFFFu);
  amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  const uint32_t sb = scale_byte(amax);
  const float mul = inv_scale(sb);
  const float sv = sb == 0xFFu ? __uint_as_float(kNaNf32) : scale_value(sb);
#pragma unroll
  for (int j = 0; j < 8; ++j) q[j] = e2m1_rn_value(w[j] * mul) * sv;
}

template <bool WINDOW_END>
__global__ void __launch_bounds__(kOscThreads)
    k_osc_step(float* __restrict__ w, float* __restrict__ w_snap,
               float* __restrict__ d_w, float* __restrict__ d_q,
               int64_t n_groups, float threshold,
               unsigned long long* __restrict__ n_flagged) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const int64_t warp = (int64_t(blockIdx.x) * kOscThreads + threadIdx.x) >> 5;
  const int64_t chunk = (int64_t(gridDim.x) * kOscThreads) >> 2;
  const int64_t my = warp * 8 + (lane >> 2);
  unsigned count = 0;
  for (int64_t base = 0; base < n_groups; base += chunk) {
    const int64_t g = base + my;
    const bool ok = g < n_groups;
    const int64_t e = (ok ? g : 0) * 32 + sub * 8;
    float vw[8], vs[8], dw[8], dq[8], qw[8], qs[8];
    load8(w + e, vw);
    load8(w_snap + e, vs);
    load8(d_w + e, dw);
    load8(d_q + e, dq);
    dq8(vw, qw);
    dq8(vs, qs);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      dw[j] = __fadd_rn(dw[j], fabsf(__fsub_rn(vw[j], vs[j])));
      dq[j] = __fadd_rn(dq[j], fabsf(__fsub_rn(qw[j], qs[j])));
    }
    if (!ok) continue;
    if (WINDOW_END) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool flag = dq[j] > __fmul_rn(threshold, dw[j]);
        if (flag) vw[j] = qw[j];
        count += flag ? 1u : 0u;
        dw[j] = 0.0f;
        dq[j] = 0.0f;
      }
      store8(w + e, vw);
    }
    store8(w_snap + e, vw);
    store8(d_w + e, dw);
    store8(d_q + e, dq);
  }
  if (WINDOW_END && n_flagged != nullptr) {
    __shared__ unsigned block_count;
    if (threadIdx.x == 0) block_count = 0;
    __syncthreads();
    count = __reduce_add_sync(0xFFFFFFFFu, count);
    if (lane == 0 && count) atomicAdd(&block_count, count);
    __syncthreads();
    if (threadIdx.x == 0 && block_count)
      atomicAdd(n_flagged, static_cast<unsigned long long>(block_count));
  }
}

// Q-Ramping ("Oscillation-Reduced MXFP4 Training for Vision Transformers",
// rebuttal, Weakness 2 and the hyper-parameter answers): one iteration.
// FLUSH (iteration 0 of an epoch): a flagged weight takes what it still
// holds, flags clear and the tracking window starts. Then the update: an
// unflagged weight takes delta at once, a flagged one gathers it and takes
// the gathered sum when APPLY (iteration % k2 == k2 - 1). TRACK (inside the
// window): the tracker's accumulation on the updated weight; WEND (the
// window's last iteration): flag d_q > k1 * d_w, reset the distances. Four
// threads per 1x32 group (the group maxima of DQ come from quad shuffles);
// every update is one fp32 operation with explicit rounding.
template <bool FLUSH, bool TRACK, bool WEND, bool APPLY>
__global__ void __launch_bounds__(kOscThreads)
    k_qramp_step(float* __restrict__ w, const float* __restrict__ delta,
                 float* __restrict__ w_snap, float* __restrict__ d_w,
                 float* __restrict__ d_q, float* __restrict__ acc,
                 uint8_t* __restrict__ flag, int64_t n_groups, float k1,
                 unsigned long long* __restrict__ n_flagged) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const int64_t warp = (int64_t(blockIdx.x) * kOscThreads + threadIdx.x) >> 5;
  const int64_t chunk = (int64_t(gridDim.x) * kOscThreads) >> 2;
  const int64_t my = warp * 8 + (lane >> 2);
  unsigned count = 0;
  for (int64_t base = 0; base < n_groups; base += chunk) {
    const int64_t g = base + my;
    const bool ok = g < n_groups;
    const int64_t e = (ok ? g : 0) * 32 + sub * 8;
    float vw[8], dv[8], va[8];
    load8(w + e, vw);
    load8(delta + e, dv);
    load8(acc + e, va);
    const uint2 f8 = *reinterpret_cast<const uint2*>(flag + e);
    uint8_t fl[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      fl[j] = uint8_t(f8.x >> (8 * j));
      fl[4 + j] = uint8_t(f8.y >> (8 * j));
    }
    float vs[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (FLUSH) {
        if (fl[j]) vw[j] = __fadd_rn(vw[j], va[j]);
        va[j] = 0.0f;
        fl[j] = 0;
        vs[j] = vw[j];
      }
      if (fl[j]) {
        va[j] = __fadd_rn(va[j], dv[j]);
        if (APPLY) {
          vw[j] = __fadd_rn(vw[j], va[j]);
          va[j] = 0.0f;
        }
      } else {
        vw[j] = __fadd_rn(vw[j], dv[j]);
      }
    }
    if (TRACK) {
      float dw[8], dq[8], qw[8], qs[8];
      if (FLUSH) {
#pragma unroll
        for (int j = 0; j < 8; ++j) dw[j] = dq[j] = 0.0f;
      } else {
        load8(w_snap + e, vs);
        load8(d_w + e, dw);
        load8(d_q + e, dq);
      }
      dq8(vw, qw);
      dq8(vs, qs);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        dw[j] = __fadd_rn(dw[j], fabsf(__fsub_rn(vw[j], vs[j])));
        dq[j] = __fadd_rn(dq[j], fabsf(__fsub_rn(qw[j], qs[j])));
        if (WEND) {
          fl[j] = dq[j] > __fmul_rn(k1, dw[j]) ? 1 : 0;
          count += ok ? fl[j] : 0u;  // threads past the last group redo group 0
          dw[j] = dq[j] = 0.0f;
        }
      }
      if (ok) {
        store8(w_snap + e, vw);
        store8(d_w + e, dw);
        store8(d_q + e, dq);
      }
    } else if (FLUSH && ok) {
      const float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      store8(w_snap + e, vs);  // the window starts from the pre-update
      store8(d_w + e, z);      // weight, but no window runs
      store8(d_q + e, z);
    }
    if (!ok) continue;
    store8(w + e, vw);
    store8(acc + e, va);
    uint2 o;
    o.x = uint32_t(fl[0]) | (uint32_t(fl[1]) << 8) | (uint32_t(fl[2]) << 16) | (uint32_t(fl[3]) << 24);
    o.y = uint32_t(fl[4]) | (uint32_t(fl[5]) << 8) | (uint32_t(fl[6]) << 16) | (uint32_t(fl[7]) << 24);
    *reinterpret_cast<uint2*>(flag + e) = o;
  }
  if (WEND && n_flagged != nullptr) {
    __shared__ unsigned block_count;
    if (threadIdx.x == 0) block_count = 0;
    __syncthreads();
    count = __reduce_add_sync(0xFFFFFFFFu, count);
    if (lane == 0 && count) atomicAdd(&block_count, count);
    __syncthreads();
    if (threadIdx.x == 0 && block_count)
      atomicAdd(n_flagged, static_cast<unsigned long long>(block_count));
  }
}

// w += s * (rel_step * |w|), s = -1 iff bit 31 of the element's hash is set.
__global__ void __launch_bounds__(kOscThreads)
    k_osc_update(float* __restrict__ w, int64_t n, RngKey key, float rel_step) {
  const int64_t n4 = n / 4;
  const int64_t stride = int64_t(gridDim.x) * kOscThreads;
  for (int64_t q = int64_t(blockIdx.x) * kOscThreads + threadIdx.x; q < n4;
       q += stride) {
    float4 v = reinterpret_cast<float4*>(w)[q];
    float* f = reinterpret_cast<float*>(&v);
    const uint64_t i0 = uint64_t(q) * 4;
    const uint32_t kh = inner_key(key, uint32_t(i0 >> 32));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t h = mix32_d(kh + uint32_t(i0) + j);
      const float mag = __fmul_rn(rel_step, fabsf(f[j]));
      f[j] = __fadd_rn(f[j], (h >> 31) ? -mag : mag);
    }
    reinterpret_cast<float4*>(w)[q] = v;
  }
  if (blockIdx.x == 0 && threadIdx.x < n - n4 * 4) {
    const uint64_t i = uint64_t(n4) * 4 + threadIdx.x;
    const uint32_t h = mix32_d(inner_key(key, uint32_t(i >> 32)) + uint32_t(i));
    const float mag = __fmul_rn(rel_step, fabsf(w[i]));
    w[i] = __fadd_rn(w[i], (h >> 31) ? -mag : mag);
  }
}

}  // namespace

cudaError_t launch_osc_step(float* w, float* w_snap, float* d_w, float* d_q,
                            int64_t rows, int64_t cols, bool window_end,
                            float threshold, unsigned long long* n_flagged,
                            cudaStream_t s) {
  const int64_t n_groups = rows * cols / kGroup;
  const int64_t blocks = (n_groups + kOscThreads / 4 - 1) / (kOscThreads / 4);
  if (window_end) {
    auto kern = k_osc_step<true>;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     kOscThreads, 0, blocks);
    kern<<<grid, kOscThreads, 0, s>>>(w, w_snap, d_w, d_q, n_groups, threshold,
                                      n_flagged);
  } else {
    auto kern = k_osc_step<false>;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     kOscThreads, 0, blocks);
    kern<<<grid, kOscThreads, 0, s>>>(w, w_snap, d_w, d_q, n_groups, threshold,
                                      n_flagged);
  }
  return cudaGetLastError();
}

template <bool FLUSH, bool TRACK, bool WEND, bool APPLY>
static cudaError_t qramp_impl(float* w, const float* delta, float* w_snap, float* d_w,
                              float* d_q, float* acc, uint8_t* flag, int64_t n_groups,
                              float k1, unsigned long long* n_flagged, cudaStream_t s) {
  auto kern = k_qramp_step<FLUSH, TRACK, WEND, APPLY>;
  const int64_t blocks = (n_groups + kOscThreads / 4 - 1) / (kOscThreads / 4);
  const int grid = persistent_grid(reinterpret_cast<const void*>(kern), kOscThreads, 0, blocks);
  kern<<<grid, kOscThreads, 0, s>>>(w, delta, w_snap, d_w, d_q, acc, flag, n_groups, k1,
                                    n_flagged);
  return cudaGetLastError();
}

template <bool FLUSH, bool TRACK, bool WEND>
static cudaError_t qramp_apply(bool apply, float* w, const float* delta, float* w_snap,
                               float* d_w, float* d_q, float* acc, uint8_t* flag,
                               int64_t n_groups, float k1, unsigned long long* n_flagged,
                               cudaStream_t s) {
  return apply ? qramp_impl<FLUSH, TRACK, WEND, true>(w, delta, w_snap, d_w, d_q, acc, flag,
                                                      n_groups, k1, n_flagged, s)
               : qramp_impl<FLUSH, TRACK, WEND, false>(w, delta, w_snap, d_w, d_q, acc, flag,
                                                       n_groups, k1, n_flagged, s);
}

cudaError_t launch_qramp_step(float* w, const float* delta, float* w_snap, float* d_w,
                              float* d_q, float* acc, uint8_t* flag, int64_t rows,
                              int64_t cols, int64_t iter, int64_t track_iters, float k1,
                              int64_t k2, unsigned long long* n_flagged, cudaStream_t s) {
  const int64_t n_groups = rows * cols / kGroup;
  const bool flush = iter == 0, track = iter < track_iters;
  const bool wend = iter == track_iters - 1, apply = iter % k2 == k2 - 1;
  if (flush) {
    if (!track)
      return qramp_apply<true, false, false>(apply, w, delta, w_snap, d_w, d_q, acc, flag,
                                             n_groups, k1, n_flagged, s);
    return wend ? qramp_apply<true, true, true>(apply, w, delta, w_snap, d_w, d_q, acc, flag,
                                                n_groups, k1, n_flagged, s)
                : qramp_apply<true, true, false>(apply, w, delta, w_snap, d_w, d_q, acc, flag,
                                                 n_groups, k1, n_flagged, s);
  }
  if (!track)
    return qramp_apply<false, false, false>(apply, w, delta, w_snap, d_w, d_q, acc, flag,
                                            n_groups, k1, n_flagged, s);
  return wend ? qramp_apply<false, true, true>(apply, w, delta, w_snap, d_w, d_q, acc, flag,
                                               n_groups, k1, n_flagged, s)
              : qramp_apply<false, true, false>(apply, w, delta, w_snap, d_w, d_q, acc, flag,
                                                n_groups, k1, n_flagged, s);
}

cudaError_t launch_osc_update(float* w, int64_t n, uint64_t seed,
                              uint32_t step, float rel_step, cudaStream_t s) {
  const RngKey key = make_key(seed + (uint64_t(step) << 32), 2);
  const int64_t blocks = (n / 4 + kOscThreads - 1) / kOscThreads;
  const int grid = persistent_grid(reinterpret_cast<const void*>(k_osc_update),
                                   kOscThreads, 0, blocks < 1 ? 1 : blocks);
  k_osc_update<<<grid, kOscThreads, 0, s>>>(w, n, key, rel_step);
  return cudaGetLastError();
}

}  // namespace mxfp4
