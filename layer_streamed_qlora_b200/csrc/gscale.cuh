// Power-of-two gradient scale for fp16 gradient tensors.
//
// Gradients reaching a layer can be tiny (the mean cross-entropy divides by
// the token count), far below fp16's normal range, so fp16 gradient storage
// is scaled: given amax = max |dh2| of the layer's mid residual gradient, the
// scale is 2^k with k chosen so that amax * 2^k lies in [2^5, 2^6).  The
// projections' row sums cannot amplify that by more than ~2^9 for these
// weight magnitudes, so nothing overflows fp16 (65504), and values 2^20 below
// the maximum are still normal fp16 numbers.  Scaling and unscaling by a
// power of two are exact.
#pragma once

__device__ __forceinline__ float grad_scale_from_amax(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 1.f;
  int e = 0;
  frexpf(amax, &e);  // amax = m * 2^e, m in [0.5, 1)
  int k = 6 - e;
  k = k < -60 ? -60 : (k > 60 ? 60 : k);
  return ldexpf(1.f, k);
}
