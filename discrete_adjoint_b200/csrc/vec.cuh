// vec.cuh -- a fixed-width register vector: K independent values of one
// scalar type, element-wise arithmetic.  A thread that carries K trajectories
// writes its step code once in terms of vec<T, K>; every operation becomes K
// independent instructions, which the scheduler can overlap (instruction-level
// parallelism K times that of one trajectory).  Each element is computed with
// exactly the scalar operation, so results are bitwise those of K = 1.
#pragma once

#include "common.cuh"

namespace gs {

template <typename T, int K>
struct vec {
  T e[K];
};

template <typename T, int K>
__device__ __forceinline__ vec<T, K> vsplat(T x) {
  vec<T, K> r;
#pragma unroll
  for (int q = 0; q < K; ++q) r.e[q] = x;
  return r;
}

#define GS_VEC_BINOP(OP)                                                                      \
  template <typename T, int K>                                                                \
  __device__ __forceinline__ vec<T, K> operator OP(const vec<T, K>& a, const vec<T, K>& b) { \
    vec<T, K> r;                                                                              \
    _Pragma("unroll") for (int q = 0; q < K; ++q) r.e[q] = a.e[q] OP b.e[q];                  \
    return r;                                                                                 \
  }                                                                                           \
  template <typename T, int K>                                                                \
  __device__ __forceinline__ vec<T, K> operator OP(T a, const vec<T, K>& b) {                 \
    vec<T, K> r;                                                                              \
    _Pragma("unroll") for (int q = 0; q < K; ++q) r.e[q] = a OP b.e[q];                       \
    return r;                                                                                 \
  }                                                                                           \
  template <typename T, int K>                                                                \
  __device__ __forceinline__ vec<T, K> operator OP(const vec<T, K>& a, T b) {                 \
    vec<T, K> r;                                                                              \
    _Pragma("unroll") for (int q = 0; q < K; ++q) r.e[q] = a.e[q] OP b;                       \
    return r;                                                                                 \
  }
GS_VEC_BINOP(+)
GS_VEC_BINOP(-)
GS_VEC_BINOP(*)
#undef GS_VEC_BINOP

template <typename T, int K>
__device__ __forceinline__ vec<T, K> operator-(const vec<T, K>& a) {
  vec<T, K> r;
#pragma unroll
  for (int q = 0; q < K; ++q) r.e[q] = -a.e[q];
  return r;
}

template <typename T, int K>
__device__ __forceinline__ vec<T, K>& operator+=(vec<T, K>& a, const vec<T, K>& b) {
#pragma unroll
  for (int q = 0; q < K; ++q) a.e[q] += b.e[q];
  return a;
}

template <typename T, int K>
__device__ __forceinline__ vec<T, K> fmaT(const vec<T, K>& a, const vec<T, K>& b, const vec<T, K>& c) {
  vec<T, K> r;
#pragma unroll
  for (int q = 0; q < K; ++q) r.e[q] = fmaT(a.e[q], b.e[q], c.e[q]);
  return r;
}

template <typename T, int K>
__device__ __forceinline__ vec<T, K> fmaT(T a, const vec<T, K>& b, const vec<T, K>& c) {
  vec<T, K> r;
#pragma unroll
  for (int q = 0; q < K; ++q) r.e[q] = fmaT(a, b.e[q], c.e[q]);
  return r;
}

}  // namespace gs
