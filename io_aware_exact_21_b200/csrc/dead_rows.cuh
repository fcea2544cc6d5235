// dead_rows.cuh -- zeroing the rows of a shared-memory tile that lie past a
// packed batch's last sequence (see first_dead_row in schedule.cuh).
#pragma once

#include <stdint.h>

namespace fa {

// Zero rows [r0, 128) of a 128-row tile of `nbox` boxes of 128-byte rows
// (box b at tile + b * 16 KB, row r at + r * 128; whole 128-byte rows, so the
// swizzle within a row does not matter), `nthr` threads from `tid` on; then
// make the stores visible to the tensor core's (async-proxy) reads.
__device__ __forceinline__ void zero_tile_rows(uint8_t* tile, int nbox, int r0, int tid, int nthr) {
    const int per_row = nbox * 8;                 // 16-byte chunks per row
    const int total = (128 - r0) * per_row;
    for (int x = tid; x < total; x += nthr) {
        const int q = x / per_row;
        const int rem = x - q * per_row;
        *reinterpret_cast<uint4*>(tile + (rem >> 3) * 16384 + (r0 + q) * 128 + (rem & 7) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// A producer's record of which ring slots had their latest load land on the
// slot's landing barrier (a tile with rows past the batch end, which a fixer
// warp zeroes before it arrives on the slot's full barrier) and the parity of
// that landing, so that a producer that gives up can wait for exactly the
// copies still in flight.
struct LandTrack {
    uint32_t dead = 0;   // bit s: the latest load into slot s landed on land[s]
    uint32_t par = 0;    // bit s: loads that landed on land[s] so far, mod 2
    __device__ __forceinline__ void note(int slot, bool to_land) {
        if (to_land) {
            dead |= 1u << slot;
            par ^= 1u << slot;
        } else {
            dead &= ~(1u << slot);
        }
    }
    __device__ __forceinline__ bool landed(int slot) const { return (dead >> slot) & 1u; }
    // parity of the latest landing on land[slot]
    __device__ __forceinline__ uint32_t land_parity(int slot) const { return ((par >> slot) & 1u) ^ 1u; }
};

}  // namespace fa
