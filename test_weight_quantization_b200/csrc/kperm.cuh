// kperm.cuh — channel order of the prepared activations.
#pragma once

namespace ttq {

// Position p of a 16-channel span of the prepared activations holds channel
// k_perm<PERM>(p) of that span. For 2-, 4- and 8-bit codes the dequantiser
// turns one shifted code word into an fp16 pair (q_c, q_c') whose channels
// lie 8, 4 or 2 apart; the activations are stored in the same order so the
// tensor-core products pair the right operands. Other widths keep the
// natural order.
template <int PERM>
__host__ __device__ constexpr int k_perm(int p) {
  return PERM == 2   ? (p >> 1) + 8 * (p & 1)
         : PERM == 4 ? 8 * (p >> 3) + ((p & 7) >> 1) + 4 * (p & 1)
         : PERM == 8 ? 4 * (p >> 2) + ((p & 3) >> 1) + 2 * (p & 1)
                     : p;
}

}  // namespace ttq
