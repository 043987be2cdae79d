// internal.h -- host helpers shared by the two kernels of libssa (not part of
// the C ABI).
#pragma once
#include <cuda.h>

namespace ssa {

// [B, L, H, d] bf16 -> 4-D TMA tensor map (d, H, L, B) with a (64, 1, rows, 1)
// box and 128-byte swizzle; coordinates past the tensor read zeros.
bool tma_map_bf16(CUtensorMap* map, const void* base, int B, int L, int H, int d, int rows);

// The per-device status word that a timed-out bounded device wait raises
// (ssa_device_status reads and clears it); nullptr on failure.
int* device_status_word(int dev);

// The current limit of one device-side wait (ssa_set_wait_timeout_ns).
unsigned long long wait_timeout_ns();

}  // namespace ssa
