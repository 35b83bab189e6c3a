// Host-side helpers shared by the libzb entry points: argument checks, device
// information, the per-device status word, and TMA tensor-map encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/zb.h"

namespace zb {

struct DeviceInfo {
    int device;
    int sm_count;
    int* status;  // device address of this device's status word
};

// Device of the calling thread; ZB_ERR_DEVICE unless it is an sm_100 part.
zb_status current_device(DeviceInfo* out);

// Bounded-wait limit for device-side spin loops (ns); ZB_WAIT_TIMEOUT_NS overrides.
unsigned long long wait_timeout_ns();

// 3-D bf16 tensor map over a [outer][rows][inner] row-major tensor, box of
// `box_rows` x `inner` elements, 128-byte swizzle, zero fill out of bounds.
zb_status make_map_bf16_3d(CUtensorMap* map, const void* base, int inner, long long rows,
                           int outer, int box_rows);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline long long n_tiles(const zb_shape& s) { return (s.n_tokens + s.tile - 1) / s.tile; }

// Common checks on a zb_shape: sizes, supported head_dim and tile.
inline zb_status check_shape(const zb_shape& s) {
    if (s.heads < 1 || s.n_tokens < 1) return ZB_ERR_SHAPE;
    if (s.head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (s.tile != 64 && s.tile != 128) return ZB_ERR_UNSUPPORTED;
    if (s.n_tokens > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    return ZB_OK;
}

}  // namespace zb
