// fa_host.h -- host-side helpers shared by the translation units of libfa.so (defined in
// fa_fwd.cu): per-device state and probing, pointer checks, TMA tensor-map encoding and a
// zero-fill launch.  Internal to the library; not part of the C ABI.
#pragma once

#include <cstddef>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

namespace fa_host {

// Forward instantiations with per-device launch state: slots 0-6 bf16 and 8-14 fp16 (one per
// head dim), 15, 17 and 18 the FP8 ones (d = 128, 64, 256), 16 the failure-path test build.
// (The backward keeps its own state in fa_bwd.cu.)
constexpr int kNumCfgSlots = 19;
constexpr int kFp8Slot = 15;
constexpr int kFaultSlot = 16;
constexpr int kFp8Slot64 = 17;
constexpr int kFp8Slot256 = 18;

constexpr int kMaxDevices = 64;
constexpr int kMaxSplits = 256;

struct DeviceState {
    bool probed = false;
    bool supported = false;
    int num_sms = 0;
    int *status_ptr = nullptr;
    bool smem_attr_set[kNumCfgSlots] = {};
    int regs_ok[kNumCfgSlots] = {};   // 0 unknown, 1 verified, -1 mismatch
};

extern std::mutex g_mutex;   // guards the per-device state and lazily found addresses

// The current device's state, probed once (sm_100 or not, SM count, status word address).
int current_device(DeviceState **out, int *dev_out);
// `bytes` starting at `p` must be device (or managed) memory of device `dev`, inside one allocation.
int check_device_range(const void *p, size_t bytes, int dev);
bool overlaps(const void *a, size_t na, const void *b, size_t nb);
// 4-D view (d, H, N, B) of a [B, N, H, d] tensor, box (cw, heads, rows, 1); elem: 0 bf16,
// 1 fp16, 2 E4M3 bytes.
int encode_bnhd(CUtensorMap *m, const void *base, int d, int H, int N, int B, int cw, int rows, int heads = 1,
                int elem = 0);
// Zero `bytes` (a multiple of 16) at dst and set n_lse floats at lse (if not NULL) to -inf.
int zero_fill(void *dst, size_t bytes, float *lse, size_t n_lse, int num_sms, cudaStream_t st);

}  // namespace fa_host
