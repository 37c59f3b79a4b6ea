// si_keys.cuh -- 64-bit selection keys.
//
// The selection order of the indexer top-k is: higher score first, and for
// equal scores the lower key index first.  Packing a (score, index) pair as
//     key = ord(score) << 32 | (0xFFFFFFFF - index)
// with ord() the order-preserving map of IEEE fp32 onto uint32 makes that
// order the plain unsigned order of the keys, so every comparison, threshold
// and merge in the kernels is one 64-bit compare and ties are resolved
// exactly.  Padding (index -1, score -inf) packs to a key below every real
// one.  -0.0 is first turned into +0.0 so that equal scores pack equally.
#pragma once
#include <cstdint>

namespace si {

__device__ __forceinline__ float canonical_score(float s) { return s + 0.0f; }

__device__ __forceinline__ uint32_t ord_f32(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float unord_f32(uint32_t o) {
    const uint32_t u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
    return __uint_as_float(u);
}

__device__ __forceinline__ uint64_t pack_key(float score, uint32_t index) {
    return (static_cast<uint64_t>(ord_f32(canonical_score(score))) << 32) | static_cast<uint64_t>(~index);
}

__device__ __forceinline__ int32_t key_index(uint64_t key) {
    return static_cast<int32_t>(~static_cast<uint32_t>(key));
}

__device__ __forceinline__ float key_score(uint64_t key) { return unord_f32(static_cast<uint32_t>(key >> 32)); }

}  // namespace si
