// Element-wise activations applied to each shard's slice of the hidden
// layer.  The pairing lets them run locally because they are element-wise
// ("Tensor parallel math", "The MLP block: column then row, one
// all-reduce").  GELU is the tanh form; Swish is SiLU (beta = 1),
// "Tensor Parallelism Explained" section 2.B.
#pragma once

#include <cmath>

namespace tpk {

enum ActKind : int { kActGeluTanh = 0, kActSwiglu = 1, kActIdentity = 2, kActRelu = 3 };

__device__ __forceinline__ float gelu_tanh_f32(float h) {
  const float kSqrt2OverPi = 0.7978845608028654f;
  const float u = kSqrt2OverPi * (h + 0.044715f * h * h * h);
  return 0.5f * h * (1.0f + tanhf(u));
}

__device__ __forceinline__ float silu_f32(float h) { return h / (1.0f + expf(-h)); }

// Hardware tanh (PTX tanh.approx.f32, one MUFU operation, relative error
// about 2^-11): used where the result is stored as bf16 (8 significant bits).
// Its absolute error (about 2^-11 near |tanh| = 1) is below the storage
// rounding of the activation except where 1 + tanh cancels (GELU of
// h below about -2, a value near zero with a tiny absolute error).
__device__ __forceinline__ float tanh_mufu(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float gelu_tanh_mufu(float h) {
  const float kSqrt2OverPi = 0.7978845608028654f;
  const float u = kSqrt2OverPi * (h + 0.044715f * h * h * h);
  return 0.5f * h * (1.0f + tanh_mufu(u));
}

// SiLU(h) = h * sigmoid(h), with sigmoid(h) = (1 + tanh(h / 2)) / 2.
__device__ __forceinline__ float silu_mufu(float h) { return h * (0.5f + 0.5f * tanh_mufu(0.5f * h)); }

__device__ __forceinline__ float act_unary_mufu(int act, float h) {
  if (act == kActGeluTanh) return gelu_tanh_mufu(h);
  if (act == kActRelu) return fmaxf(h, 0.0f);
  return h;
}

// Derivatives for the backward pass (results are stored as bf16).
// d/dh GELU_tanh = 0.5 (1 + tanh u) + 0.5 h (1 - tanh^2 u) u', u = c (h + 0.044715 h^3).
__device__ __forceinline__ float gelu_tanh_grad_mufu(float h) {
  const float kSqrt2OverPi = 0.7978845608028654f;
  const float h2 = h * h;
  const float t = tanh_mufu(kSqrt2OverPi * (h + 0.044715f * h2 * h));
  const float du = kSqrt2OverPi * (1.0f + 3.0f * 0.044715f * h2);
  return 0.5f * (1.0f + t) + 0.5f * h * (1.0f - t * t) * du;
}

// sigmoid(h) = (1 + tanh(h / 2)) / 2; d/dh SiLU = sigmoid (1 + h (1 - sigmoid)).
__device__ __forceinline__ float sigmoid_mufu(float h) { return 0.5f + 0.5f * tanh_mufu(0.5f * h); }

__device__ __forceinline__ float act_grad_unary_mufu(int act, float h) {
  if (act == kActGeluTanh) return gelu_tanh_grad_mufu(h);
  if (act == kActRelu) return h > 0.0f ? 1.0f : 0.0f;
  return 1.0f;
}

// Single-input activations (GELU / identity / ReLU).
__device__ __forceinline__ float act_unary(int act, float h) {
  if (act == kActGeluTanh) return gelu_tanh_f32(h);
  if (act == kActRelu) return fmaxf(h, 0.0f);
  return h;
}

}  // namespace tpk
