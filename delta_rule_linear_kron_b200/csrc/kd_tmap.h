// kd_tmap.h -- host helper: TMA tensor maps over [B, T, H, D] activations.
#pragma once

#include <cuda.h>

namespace kd {

// Encodes a 4-D tiled TMA descriptor for a contiguous [B, T, H, D] tensor of
// element size es (2 = bf16, 4 = fp32).  Dimensions innermost first
// (D, H, T, B); the box is (box_d channels, 1 head, 64 positions, 1 batch), so
// a chunk whose positions run past T is zero-filled instead of reading the
// next sequence.  swizzle128 selects the 128-byte swizzle (box_d * es must be
// 128).  Returns false if the driver rejects the descriptor.
bool make_tmap_bthd(CUtensorMap* m, const void* base, int es, int B, int T, int H, int D, int box_d,
                    bool swizzle128);

}  // namespace kd
