// sm100_bulk.cuh -- PTX wrappers for untiled bulk copies and byte permutes (sm_100a),
// used by the GEMM and the dequantiser.
#pragma once

#include <cstdint>

namespace mxq {
namespace ptx {

// Untiled bulk copy global -> shared (both 16-byte aligned, a multiple of 16 bytes),
// completing on an mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(pol)
        : "memory");
}

__device__ __forceinline__ uint32_t ld_shared_u8(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// Byte permute: byte i of the result is byte (sel nibble i) of {b, a} (a = bytes 0-3).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Eight E2M1 codes (nibbles of cw, code 2i in the low nibble of byte i) -> eight bf16
// values, two per word (even code in the low half).  The bf16 bits of the magnitudes
// {0, 0.5, 1, 1.5, 2, 3, 4, 6} are 00 00 / 3F 00 / 3F 80 / 3F C0 / 40 00 / 40 40 / 40 80 /
// 40 C0: two byte permutes pick the high and the low bytes by the 3-bit magnitude index
// (a selector reads only the low four nibbles), two more interleave them.  The signs: bit
// 3 of code 2j sits at bit 7 of byte j of (cw & 0x88888888) << 4, bit 3 of code 2j + 1 at
// bit 7 of byte j of cw & 0x88888888; one permute per word moves them to bits 15 and 31.
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t cw, uint32_t (&w)[4])
{
    const uint32_t m = cw & 0x77777777u, mh = m >> 16;
    const uint32_t h0 = prmt(0x3F3F3F00u, 0x40404040u, m), l0 = prmt(0xC0800000u, 0xC0804000u, m);
    const uint32_t h1 = prmt(0x3F3F3F00u, 0x40404040u, mh), l1 = prmt(0xC0800000u, 0xC0804000u, mh);
    const uint32_t sg = cw & 0x88888888u, sl = sg << 4;
    w[0] = prmt(l0, h0, 0x5140u) | (prmt(sl, sg, 0x4000u) & 0x80008000u);
    w[1] = prmt(l0, h0, 0x7362u) | (prmt(sl, sg, 0x5010u) & 0x80008000u);
    w[2] = prmt(l1, h1, 0x5140u) | (prmt(sl, sg, 0x6020u) & 0x80008000u);
    w[3] = prmt(l1, h1, 0x7362u) | (prmt(sl, sg, 0x7030u) & 0x80008000u);
}

}  // namespace ptx
}  // namespace mxq

namespace mxq {
namespace ptx {

// Wait until at most N bulk async-groups of this thread are still reading their source.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

}  // namespace ptx
}  // namespace mxq

namespace mxq {
namespace ptx {

// 16-byte asynchronous copy global -> shared (both 16-byte aligned), tracked per thread by
// commit/wait groups.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace ptx
}  // namespace mxq
