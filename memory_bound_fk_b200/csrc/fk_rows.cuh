// fk_rows.cuh -- register-resident row I/O shared by the row kernels
// (softmax, LayerNorm): a team of TEAM threads (a warp or a block) covers a
// row, or a slice of it, in chunks of TEAM 16-byte vectors.  On the vector
// path thread t owns vector (chunk * TEAM + t), so a warp's loads are 512
// contiguous bytes; when rows or pointers are not 16-byte aligned, the
// scalar path keeps the same chunks but gives thread t the elements
// chunk*TEAM*VEC + k*TEAM + t (k < VEC), again contiguous per warp.
#pragma once

#include <stdint.h>

#include "fk_common.cuh"

namespace fk {
namespace {

template <typename I>
__device__ __forceinline__ I imin(I a, I b) {
  return a < b ? a : b;
}

// Load VPT chunks of a team slice as raw 16-byte words (VPT * VEC values).
// Vectors [vfirst, ve) of the row are the slice; anything outside is -inf.
// MASK: elements at or after `lim` are -inf too and are not loaded.
// ZERO: the fill is +0 instead of -inf (sums rather than maxima).
// The scalar (unaligned) path packs its scalar loads into the same layout.
template <typename T, int VPT, int TEAM, bool ALIGNED, bool MASK, typename Idx, bool ZERO = false>
__device__ __forceinline__ void load_chunks(const T* row, Idx vfirst, Idx ve, Idx cols, Idx lim, int t,
                                            uint4* raw) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr uint32_t kFill = ZERO ? 0u : Elem<T>::kNegInfWord;
  const float fill = ZERO ? 0.0f : -INFINITY;
  if constexpr (ALIGNED) {
#pragma unroll
    for (int c = 0; c < VPT; ++c) {
      const Idx vi = vfirst + static_cast<Idx>(c) * TEAM + t;
      const bool live = MASK ? (vi < ve && vi * VEC < lim) : (vi < ve);
      raw[c] = ld_stream_v4_if(row + static_cast<size_t>(vi) * VEC, live, kFill);
    }
    // Vectors wholly past lim were not loaded (all -inf); only the one that
    // straddles lim needs its tail masked.  One thread of the team holds it,
    // so the masking sits behind a warp vote: masking every vector in the
    // unrolled loop (the selects run for all of them) added 40% to the
    // instructions of causal 2048-column rows and made them issue-bound.
    // Every caller runs this with all lanes of the warp converged.
    if constexpr (MASK) {
      const Idx vs = lim / VEC;  // the straddling vector, if lim % VEC != 0
      const Idx off = vs - vfirst;
      const bool mine = (lim % VEC != 0) && vs >= vfirst && vs < ve && off / TEAM < static_cast<Idx>(VPT) &&
                        off % TEAM == static_cast<Idx>(t);
      if (__any_sync(0xffffffffu, mine) && mine) {
        const int cs = static_cast<int>(off / TEAM);
        const int keep = static_cast<int>(lim % VEC);
#pragma unroll
        for (int c = 0; c < VPT; ++c)
          if (c == cs) raw[c] = Elem<T>::keep_first(raw[c], keep);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < VPT; ++c) {
      const Idx e0 = (vfirst + static_cast<Idx>(c) * TEAM) * VEC + t;
      Idx eend = (ve * VEC < cols) ? ve * VEC : cols;
      if constexpr (MASK) eend = imin(eend, lim);
      float f[VEC];
#pragma unroll
      for (int k = 0; k < VEC; ++k) {
        const Idx e = e0 + static_cast<Idx>(k) * TEAM;
        f[k] = (e < eend) ? Elem<T>::load1(row + e) : fill;
      }
      raw[c] = Elem<T>::pack(f);  // exact: the values are already of type T
    }
  }
}

// Store, for the same placement as load_chunks, the values that
// fn(c, o) writes into o[0..VEC) for chunk c (fn is called once per chunk,
// in order, so callers can produce each chunk just before it is stored).
// WLIM: vectors (aligned path) or elements (scalar path) at or after wlim
// are not stored.
template <typename T, int VPT, int TEAM, bool ALIGNED, typename Idx, bool WLIM = false, typename Fn>
__device__ __forceinline__ void store_chunks_fn(T* row, Idx vfirst, Idx ve, Idx cols, int t, Fn fn, Idx wlim = 0) {
  constexpr int VEC = Elem<T>::VEC;
#pragma unroll
  for (int c = 0; c < VPT; ++c) {
    float o[VEC];
    fn(c, o);
    if constexpr (ALIGNED) {
      const Idx vi = vfirst + static_cast<Idx>(c) * TEAM + t;
      const bool st = WLIM ? (vi < ve && vi * VEC < wlim) : (vi < ve);
      st_stream_v4_if(row + static_cast<size_t>(vi) * VEC, Elem<T>::pack(o), st);
    } else {
      const Idx e0 = (vfirst + static_cast<Idx>(c) * TEAM) * VEC + t;
      Idx eend = (ve * VEC < cols) ? ve * VEC : cols;
      if constexpr (WLIM) eend = eend < wlim ? eend : wlim;
#pragma unroll
      for (int k = 0; k < VEC; ++k) {
        const Idx e = e0 + static_cast<Idx>(k) * TEAM;
        if (e < eend) Elem<T>::store1(row + e, o[k]);
      }
    }
  }
}

// Store v * scale for the same placement as load_chunks (WLIM: as above).
template <typename T, int VPT, int TEAM, bool ALIGNED, typename Idx, bool WLIM = false>
__device__ __forceinline__ void store_chunks(T* row, Idx vfirst, Idx ve, Idx cols, int t, const float* v,
                                             float scale, Idx wlim = 0) {
  constexpr int VEC = Elem<T>::VEC;
  store_chunks_fn<T, VPT, TEAM, ALIGNED, Idx, WLIM>(
      row, vfirst, ve, cols, t,
      [&](int c, float* o) {
#pragma unroll
        for (int k = 0; k < VEC; ++k) o[k] = v[c * VEC + k] * scale;
      },
      wlim);
}

// Row loads: raw 16-byte words; fp32 rows are unpacked into v at once (the
// same bits), bf16 rows stay packed until exp_sum.
template <typename T, int VPT, int TEAM, bool ALIGNED, bool MASK, typename Idx, bool ZERO = false>
__device__ __forceinline__ void load_row(const T* row, Idx vfirst, Idx ve, Idx cols, Idx lim, int t,
                                         uint4* raw, float* v) {
  load_chunks<T, VPT, TEAM, ALIGNED, MASK, Idx, ZERO>(row, vfirst, ve, cols, lim, t, raw);
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) Elem<T>::unpack(raw[i], v + i * Elem<T>::VEC);
  }
}

}  // namespace
}  // namespace fk
