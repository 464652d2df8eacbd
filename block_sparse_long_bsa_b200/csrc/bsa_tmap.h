// Host-side TMA tensor-map encoding shared by the kernels' launchers
// (bf16 tensors, 128-byte swizzle, out-of-bounds rows zero-filled on load and
// clipped on store).  Internal to the library.
#pragma once

#include <cuda.h>

namespace bsa {
namespace tmap {

// Fetches cuTensorMapEncodeTiled from the driver once; BSA_OK or an error
// (message set) if the driver does not provide it.
int get_encoder();

// [slices][n][d] bf16 in boxes of `rows` rows of one slice, landing in shared
// memory as [64-column atom][rows][64 columns] (for d = 128 the atom is a
// tensor dimension of stride 128 bytes, so one box holds both atoms).
int encode_rows(CUtensorMap* m, const void* ptr, int slices, int n, int d, int rows);

// K or V [kv_heads][n][d]: one 64-row chunk of one head per box.
inline int encode_kv(CUtensorMap* m, const void* ptr, int slices, int n, int d) {
  return encode_rows(m, ptr, slices, n, d, 64);
}

// Q-shaped [heads][n][d]: one 128-row tile per box -- B = 128: one block of
// one head; B = 64: the same block of two consecutive heads (the head
// dimension inside the atom dimension), landing as [atom][128 rows][64 columns].
int encode_q(CUtensorMap* m, const void* ptr, int heads, int n, int d, int blk);

// [slices][n][d] bf16 in boxes of `rows` rows x 64 columns of one slice (the
// column coordinate picks the 64-column atom), so several boxes can be
// placed as [atom][rows of several blocks][64 columns].
int encode_atoms(CUtensorMap* m, const void* ptr, int slices, int n, int d, int rows);

// o [heads][n][d] for stores: one warp's 32 rows x 64 columns per box.
int encode_o(CUtensorMap* m, const void* ptr, int heads, int n, int d);

}  // namespace tmap
}  // namespace bsa
