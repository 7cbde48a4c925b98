// qlin_common.cuh -- packed-weight layout and device helpers shared by the libqlin kernels.
#pragma once
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/qlin.h"

namespace qlin {

// ------------------------------------------------------------------ packed layout
//
// [ header 256 B ][ unit (t=0,g=0) ][ unit (0,1) ] ... [ unit (T-1, G-1) ]
//
// A tile is 32 output rows; a k-group is 256 inputs = 8 parts of 32.  One unit = (tile t,
// k-group g) is contiguous:
//   codes : 32 rows x 8 parts, 16 B per (row, part) for 4-bit formats, or 2 x 16 B for Q8_0 stored
//           as two planes [half][row][part]; vector index of (row r, part p) is r * 8 + p.
//   scales: 32 lanes x 16 B.  Lane l = (r % 4) * 8 + p holds, in slot i = r / 4, the scale(s) of
//           (row r, part p): one fp16 d (Q8_0 / Q4_0) or two E4M3 bytes (NVFP4, one per 16).
//           MXFP4: 32 lanes x 8 B, one UE8M0 byte per (row, part) in slot i.
//           Q4_K: as Q4_0, the 16-bit slot holding (row r, part p)'s 6-bit sub-block scale in
//           bits 0..5 and 6-bit min in bits 6..11; then 32 x 4 B of per-row super-block scales
//           {fp16 d, fp16 dmin}, row r at entry (r % 4) * 8 + r / 4, so lane l reads the 8 rows
//           it works on as 32 contiguous bytes at entry (l / 8) * 8.
//           Q6_K: codes as Q8_0's two planes (byte = 6-bit code, 0..63); the 16-bit slot holds the
//           int8 scales of elements 0..15 (low byte) and 16..31 (high byte); then per-row {fp16 d, 0}
//           entries as Q4_K.
// A warp reading vector (lane + 32 * i) in step i therefore touches 512 contiguous bytes, and
// lane l always works on part l % 8 of rows l / 8 + 4 i (i = 0..7).
// Element order inside a part:
//   4-bit: element e in byte e / 2, low nibble for even e (word k holds elements 8k .. 8k+7);
//          Q4_0 and Q4_K codes are stored as they are (0..15)
//   Q8_0 : element e in byte e of the 32-byte part (plane e / 16), stored as q + 128
// QLIN_PACK_GATE_UP tiles: rows 0..15 = gate rows 16 t + r, rows 16..31 = up rows N/2 + 16 t + r.
constexpr int kHdrBytes = 256;
constexpr int kTileRows = 32;
constexpr int kGroupK = 256;
constexpr int kParts = 8;
constexpr uint32_t kMagic = 0x4e494c51u;  // "QLIN"

struct PackedHeader {
    uint32_t magic;
    uint32_t fmt;
    int64_t N;
    int64_t K;
    uint32_t flags;
    float global_scale;
    int32_t T;  // tiles
    int32_t G;  // k-groups
    uint32_t unit_bytes;
    uint32_t reserved[53];
};
static_assert(sizeof(PackedHeader) == kHdrBytes, "header size");

__host__ __device__ constexpr int code_bytes(int fmt) { return (fmt == QLIN_Q8_0 || fmt == QLIN_Q6_K) ? 8192 : 4096; }
__host__ __device__ constexpr int unit_bytes(int fmt) {
    return code_bytes(fmt) + (fmt == QLIN_MXFP4 ? 256 : (fmt == QLIN_Q4_K || fmt == QLIN_Q6_K) ? 640 : 512);
}
// K-quants: 32 per-row 4-byte entries after the (row, part) slots -- Q4_K {fp16 d, fp16 dmin},
// Q6_K {fp16 d, 0} -- row r at entry (r % 4) * 8 + r / 4.
__host__ __device__ constexpr int row_d_off(int fmt) { return code_bytes(fmt) + 512; }

struct Geometry {
    int64_t T, G, U;  // tiles, k-groups, units
    int64_t Kpad;
    int rows_per_half;  // 16 for GATE_UP tiles, else 32 (output rows per tile)
};

inline Geometry geometry(int fmt, int64_t N, int64_t K, int pack_flags) {
    Geometry g;
    g.G = (K + kGroupK - 1) / kGroupK;
    g.Kpad = g.G * kGroupK;
    if (pack_flags & QLIN_PACK_GATE_UP) {
        g.T = (N / 2 + 15) / 16;
        g.rows_per_half = 16;
    } else {
        g.T = (N + kTileRows - 1) / kTileRows;
        g.rows_per_half = 32;
    }
    g.U = g.T * g.G;
    (void)fmt;
    return g;
}

// ------------------------------------------------------------------ device helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Budget of the bounded waits between CTAs (dependency counts, grid barriers, partial sums of
// other CTAs): the uint32 at byte kWsWaitBudgetOff of a workspace, in nanoseconds, or ~2 s when it
// is 0 (a zero-filled workspace).  Set with qlin_ws_set_wait_budget; read once per launch.
constexpr int64_t kWsWaitBudgetOff = 32;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
__device__ __forceinline__ uint64_t ws_wait_budget_ns(const void* ws) {
    const unsigned v = __ldcg(reinterpret_cast<const unsigned*>(reinterpret_cast<const uint8_t*>(ws) + kWsWaitBudgetOff));
    return v ? (uint64_t)v : kDefaultWaitNs;
}

// Bounded wait on an mbarrier phase: gives up after ~timeout_ns and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t timeout_ns = 2000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0 && globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// One bulk global -> shared copy completing on an mbarrier (sizes and addresses 16-B aligned).
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ float4 ldg_f4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ float fp16_bits_to_f32(uint32_t h) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// OCP E4M3 ("fn") byte -> fp32, exact (hardware conversion via the x2 form).
// OCP MX UE8M0 scale byte: 2^(b - 127) as fp32 (b = 0: the subnormal 2^-127), 0xFF = NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
    b &= 0xffu;
    if (b == 0xffu) return __uint_as_float(0x7fc00000u);
    return __uint_as_float(b == 0u ? 0x00400000u : b << 23);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    uint32_t h2;
    uint16_t in = static_cast<uint16_t>(b & 0xffu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xffffu)));
}

// Two E2M1 codes (one byte: element 2i low nibble, 2i+1 high) -> f16x2 (low half = low nibble).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t h2;
    uint16_t in = static_cast<uint16_t>(byte & 0xffu);
    asm("{\n .reg .b8 t;\n cvt.u8.u16 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}\n" : "=r"(h2) : "h"(in));
    return h2;
}

__device__ __forceinline__ uint32_t atomic_ticket(int* p) { return atomicAdd(p, 1); }

}  // namespace qlin
