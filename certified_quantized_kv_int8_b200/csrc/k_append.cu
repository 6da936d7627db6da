// Append path: seal complete 64-token blocks into Tier 1 and copy them to
// Tier 2; keep the residual (unsealed) block exact in device memory.  A token
// reaches Tier 2 when its block seals: until then only the residual block,
// never promoted, holds it, so appends of single tokens touch device memory
// alone and the host link carries whole blocks.
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §1
// (tiered storage): Tier 1 holds per-channel INT8 keys and per-group INT4
// values with their scales/offsets and per-block error annotations; Tier 2
// holds the FP16 originals in pinned host memory.
//
// Readings used (the pages give no formulas):
//   keys   s_c = amax_c / 127 over the block, code = rint(k / s) in [-127, 127]
//   values per (token, 32 channels): z = min, s = (max - min) / 15,
//          code = rint((v - z) / s) in [0, 15], v_hat = s * code + z
//   eta_b  max over the block of |v - v_hat|
// Every step is one IEEE float32 operation (explicit _rn intrinsics, never
// contracted into an FMA), so codes and annotations are reproducible bit for bit.
// With binary16 metadata (Tier1::meta16) both scales are rounded up to
// binary16 (__float2half_ru) before the codes are taken against them, so no
// code is clamped and the stored scale bounds the rounding error; the value
// offset, the min of binary16 inputs, is stored exactly.
#include "cqa_internal.cuh"

namespace cqa {

namespace {

__device__ __forceinline__ void atomic_max_f(float* a, float v) {
  if (v >= 0.f)
    atomicMax(reinterpret_cast<int*>(a), __float_as_int(v));
  else
    atomicMin(reinterpret_cast<unsigned*>(a), __float_as_uint(v));
}

__device__ __forceinline__ void atomic_min_f(float* a, float v) {
  if (v >= 0.f)
    atomicMin(reinterpret_cast<int*>(a), __float_as_int(v));
  else
    atomicMax(reinterpret_cast<unsigned*>(a), __float_as_uint(v));
}

// grid (blocks to seal, B*Hkv), 256 threads.  Block j gathers its 64 tokens
// from the old residual (tokens < T_old) and from the new input.
template <int D>
__global__ void __launch_bounds__(256) seal_kernel(Tier1 t, Strides st, int unit0,
                                                   const __half* __restrict__ knew,
                                                   const __half* __restrict__ vnew, int T_old,
                                                   int n_new, int nb_old) {
  constexpr int C8 = D / 8;  // 16-byte chunks per token row
  constexpr int NG = D / VG;
  const int j = nb_old + blockIdx.x;
  const int ug = blockIdx.y;
  const size_t u = (size_t)unit0 + ug;
  __shared__ __align__(16) __half ks[BLK * D];
  __shared__ __align__(16) __half vs[BLK * D];
  __shared__ float sc[D];
  __shared__ int eta_bits;

  for (int e = threadIdx.x; e < BLK * C8; e += blockDim.x) {
    const int tk = e / C8, c8 = e % C8;
    const int tok = j * BLK + tk;
    const uint4 *sk, *sv;
    if (tok < T_old) {
      const size_t off = u * st.res + (size_t)(tok - nb_old * BLK) * D + c8 * 8;
      sk = reinterpret_cast<const uint4*>(t.kres + off);
      sv = reinterpret_cast<const uint4*>(t.vres + off);
    } else {
      const size_t off = ((size_t)ug * n_new + (tok - T_old)) * D + c8 * 8;
      sk = reinterpret_cast<const uint4*>(knew + off);
      sv = reinterpret_cast<const uint4*>(vnew + off);
    }
    reinterpret_cast<uint4*>(ks)[e] = *sk;
    reinterpret_cast<uint4*>(vs)[e] = *sv;
  }
  if (threadIdx.x == 0) eta_bits = 0;
  __syncthreads();

  // the block's FP16 originals to Tier 2 (pinned host memory, device-mapped)
  for (int e = threadIdx.x; e < BLK * C8; e += blockDim.x) {
    const int tk = e / C8, c8 = e % C8;
    const size_t dst2 = u * st.tier2 + ((size_t)j * BLK + tk) * D + c8 * 8;
    *reinterpret_cast<uint4*>(t.k2 + dst2) = reinterpret_cast<const uint4*>(ks)[e];
    *reinterpret_cast<uint4*>(t.v2 + dst2) = reinterpret_cast<const uint4*>(vs)[e];
  }

  // per-channel key scale
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float a = 0.f;
    for (int tk = 0; tk < BLK; ++tk) a = fmaxf(a, fabsf(__half2float(ks[tk * D + c])));
    const float s = __fdiv_rn(a, 127.0f);
    sc[c] = t.meta16 ? __half2float(__float2half_ru(s)) : s;
  }
  __syncthreads();

  int8_t* kc = t.kcodes + u * st.kcodes + (size_t)j * BLK * D;
  for (int e = threadIdx.x; e < BLK * D / 4; e += blockDim.x) {
    const int tk = e / (D / 4), c0 = (e % (D / 4)) * 4;
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float s = sc[c0 + i];
      int code = 0;
      if (s > 0.f) {
        const float r = rintf(__fdiv_rn(__half2float(ks[tk * D + c0 + i]), s));
        code = (int)fminf(fmaxf(r, -127.f), 127.f);
      }
      w |= (uint32_t)(uint8_t)(int8_t)code << (8 * i);
    }
    reinterpret_cast<uint32_t*>(kc)[e] = w;
  }
  if (t.meta16) {
    __half* ksc = t.kscale_h + u * st.kscale + (size_t)j * D;
    for (int c = threadIdx.x; c < D; c += blockDim.x) ksc[c] = __float2half_rn(sc[c]);  // exact
  } else {
    float* ksc = t.kscale + u * st.kscale + (size_t)j * D;
    for (int c = threadIdx.x; c < D; c += blockDim.x) ksc[c] = sc[c];
  }

  // values: one thread per (token, group)
  uint8_t* vc = t.vcodes + u * st.vcodes + (size_t)j * BLK * (D / 2);
  const size_t vm0 = u * st.vmeta + (size_t)j * BLK * NG * 2;
  float emax = 0.f;
  for (int e = threadIdx.x; e < BLK * NG; e += blockDim.x) {
    const int tk = e / NG, gi = e % NG;
    const __half* v = vs + tk * D + gi * VG;
    float lo = __half2float(v[0]), hi = lo;
    for (int i = 1; i < VG; ++i) {
      const float x = __half2float(v[i]);
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
    float s = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
    if (t.meta16) s = __half2float(__float2half_ru(s));
    uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < VG; ++i) {
      const float x = __half2float(v[i]);
      int code = 0;
      if (s > 0.f) {
        const float r = rintf(__fdiv_rn(__fsub_rn(x, lo), s));
        code = (int)fminf(fmaxf(r, 0.f), 15.f);
      }
      const float vh = __fadd_rn(__fmul_rn(s, (float)code), lo);
      emax = fmaxf(emax, fabsf(__fsub_rn(x, vh)));
      packed[i / 8] |= (uint32_t)code << (4 * (i % 8));
    }
    *reinterpret_cast<uint4*>(vc + (size_t)tk * (D / 2) + gi * (VG / 2)) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
    const size_t mi = vm0 + (size_t)(tk * NG + gi) * 2;
    if (t.meta16) {
      t.vmeta_h[mi] = __float2half_rn(s);       // exact: s was rounded to binary16
      t.vmeta_h[mi + 1] = __float2half_rn(lo);  // exact: the min of binary16 inputs
    } else {
      t.vmeta[mi] = s;
      t.vmeta[mi + 1] = lo;
    }
  }
  atomicMax(&eta_bits, __float_as_int(emax));  // emax >= 0: int order = float order
  __syncthreads();
  if (threadIdx.x == 0) t.eta[u * st.eta + j] = __int_as_float(eta_bits);
}

// grid (ceil(n_new/64), B*Hkv), 256 threads: residual slots, per-channel
// value range, and the rows' new length (read by the decode kernels).
template <int D>
__global__ void __launch_bounds__(256) append_tail_kernel(Tier1 t, Strides st, int unit0,
                                                          const __half* __restrict__ knew,
                                                          const __half* __restrict__ vnew,
                                                          int T_old, int n_new, int nb_new,
                                                          int32_t* __restrict__ lens_rows,
                                                          int Hkv) {
  constexpr int C8 = D / 8;
  const int ug = blockIdx.y;
  const size_t u = (size_t)unit0 + ug;
  if (blockIdx.x == 0 && threadIdx.x == 0 && ug % Hkv == 0) lens_rows[ug / Hkv] = T_old + n_new;
  const int i0 = blockIdx.x * BLK;
  const int n = min(BLK, n_new - i0);
  for (int e = threadIdx.x; e < n * C8; e += blockDim.x) {
    const int i = i0 + e / C8, c8 = e % C8;
    const int tok = T_old + i;
    const size_t src = ((size_t)ug * n_new + i) * D + c8 * 8;
    if (tok >= nb_new * BLK) {
      const uint4 kv = *reinterpret_cast<const uint4*>(knew + src);
      const uint4 vv = *reinterpret_cast<const uint4*>(vnew + src);
      const size_t dr = u * st.res + (size_t)(tok - nb_new * BLK) * D + c8 * 8;
      *reinterpret_cast<uint4*>(t.kres + dr) = kv;
      *reinterpret_cast<uint4*>(t.vres + dr) = vv;
    }
  }
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float lo = INFINITY, hi = -INFINITY;
    for (int i = 0; i < n; ++i) {
      const float x = __half2float(vnew[((size_t)ug * n_new + i0 + i) * D + c]);
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
    // +0.0 for -0.0 so that the integer-ordered atomics see one zero
    atomic_min_f(t.vrange + u * st.vrange + c, __fadd_rn(lo, 0.0f));
    atomic_max_f(t.vrange + u * st.vrange + D + c, __fadd_rn(hi, 0.0f));
  }
}

}  // namespace

cudaError_t launch_seal(const Tier1& t, const Strides& st, int unit0, int B, int Hkv, int d,
                        const __half* knew, const __half* vnew, int T_old, int n_new, int nb_old,
                        int nb_new, cudaStream_t s) {
  if (nb_new <= nb_old) return cudaSuccess;
  dim3 grid(nb_new - nb_old, B * Hkv);
  if (d == 128)
    seal_kernel<128><<<grid, 256, 0, s>>>(t, st, unit0, knew, vnew, T_old, n_new, nb_old);
  else
    seal_kernel<64><<<grid, 256, 0, s>>>(t, st, unit0, knew, vnew, T_old, n_new, nb_old);
  return cudaGetLastError();
}

cudaError_t launch_append_tail(const Tier1& t, const Strides& st, int unit0, int B, int Hkv,
                               int d, const __half* knew, const __half* vnew, int T_old,
                               int n_new, int nb_new, int32_t* lens_rows, cudaStream_t s) {
  dim3 grid((n_new + BLK - 1) / BLK, B * Hkv);
  if (d == 128)
    append_tail_kernel<128><<<grid, 256, 0, s>>>(t, st, unit0, knew, vnew, T_old, n_new, nb_new,
                                                 lens_rows, Hkv);
  else
    append_tail_kernel<64><<<grid, 256, 0, s>>>(t, st, unit0, knew, vnew, T_old, n_new, nb_new,
                                                lens_rows, Hkv);
  return cudaGetLastError();
}

}  // namespace cqa
