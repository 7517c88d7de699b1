// mxq_api.cu -- the C ABI of libmxq.so (declared in include/mxq.h).
//
// Host-side layer only.  It validates arguments so that a bad call cannot reach
// the GPU: sizes, alignment, device residency and extent of every buffer,
// overlap of outputs with inputs.  It then builds the TMA descriptor over X
// and launches the kernels on the caller's stream.  It allocates no device
// memory.  The only state kept across calls is a per-thread cache of encoded TMA
// descriptors (keyed by everything a descriptor is encoded from) and, per device,
// the SM count and which kernels have their shared-memory opt-in set.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/mxq.h"
#include "mxq_internal.h"

namespace {

thread_local char g_last_error[256] = "no error";

void note_cuda(cudaError_t e, const char *where)
{
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s (%d)", where, cudaGetErrorString(e),
                  static_cast<int>(e));
}

void note_cu(CUresult r, const char *where)
{
    std::snprintf(g_last_error, sizeof g_last_error, "%s: CUresult %d", where, static_cast<int>(r));
}

// Driver entry points, fetched through the runtime (no link against libcuda).
struct Driver {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    PFN_cuPointerGetAttributes_v7000 ptr_attrs = nullptr;
    bool ok = false;
};

const Driver &driver()
{
    static Driver d;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q1, q2;
        void *p1 = nullptr, *p2 = nullptr;
        cudaError_t e1 = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p1, 12000,
                                                          cudaEnableDefault, &q1);
        cudaError_t e2 = cudaGetDriverEntryPointByVersion("cuPointerGetAttributes", &p2, 7000,
                                                          cudaEnableDefault, &q2);
        if (e1 == cudaSuccess && e2 == cudaSuccess && q1 == cudaDriverEntryPointSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            d.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p1);
            d.ptr_attrs = reinterpret_cast<PFN_cuPointerGetAttributes_v7000>(p2);
            d.ok = true;
        }
    });
    return d;
}

struct DeviceInfo {
    std::atomic<int> state{0};   // 0 unknown, 1 supported, 2 unsupported
    int num_sms = 0;
};
DeviceInfo g_dev[64];

// Resolve the current device and check it is an sm_100 part.
mxq_status current_device(int *dev_out, int *sms_out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        note_cuda(e, "cudaGetDevice");
        return MXQ_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) return MXQ_ERR_UNSUPPORTED;
    DeviceInfo &info = g_dev[dev];
    if (info.state.load(std::memory_order_acquire) == 0) {
        int major = 0, sms = 0, optin = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) {
            note_cuda(e, "cudaDeviceGetAttribute");
            return MXQ_ERR_CUDA;
        }
        info.num_sms = sms;
        info.state.store((major == 10 && optin >= 210 * 1024) ? 1 : 2, std::memory_order_release);
    }
    if (info.state.load(std::memory_order_acquire) != 1) return MXQ_ERR_UNSUPPORTED;
    *dev_out = dev;
    *sms_out = info.num_sms;
    return MXQ_OK;
}

// [p, p + bytes) must be device (or managed) memory of `dev`, inside one allocation.
mxq_status check_buffer(const void *p, uint64_t bytes, int dev)
{
    const Driver &d = driver();
    if (!d.ok) {
        std::snprintf(g_last_error, sizeof g_last_error, "driver entry points unavailable");
        return MXQ_ERR_CUDA;
    }
    unsigned int mem_type = 0;
    int ordinal = -1;
    CUdeviceptr start = 0;
    size_t size = 0;
    CUpointer_attribute attrs[4] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE, CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL,
                                    CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, CU_POINTER_ATTRIBUTE_RANGE_SIZE};
    void *data[4] = {&mem_type, &ordinal, &start, &size};
    CUresult r = d.ptr_attrs(4, attrs, data, reinterpret_cast<CUdeviceptr>(p));
    if (r != CUDA_SUCCESS) {
        note_cu(r, "cuPointerGetAttributes");
        return MXQ_ERR_INVALID_ARG;
    }
    if (mem_type != CU_MEMORYTYPE_DEVICE || ordinal != dev) {
        std::snprintf(g_last_error, sizeof g_last_error, "pointer %p is not device memory of device %d", p, dev);
        return MXQ_ERR_INVALID_ARG;
    }
    const uint64_t a = reinterpret_cast<uint64_t>(p);
    if (start != 0 && size != 0 && (a < start || a + bytes > start + size)) {
        std::snprintf(g_last_error, sizeof g_last_error, "buffer %p + %llu B overruns its allocation", p,
                      static_cast<unsigned long long>(bytes));
        return MXQ_ERR_INVALID_ARG;
    }
    return MXQ_OK;
}

bool overlaps(const void *a, uint64_t na, const void *b, uint64_t nb)
{
    const uint64_t x = reinterpret_cast<uint64_t>(a), y = reinterpret_cast<uint64_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

bool aligned(const void *p, uint64_t n) { return (reinterpret_cast<uint64_t>(p) % n) == 0; }

mxq_status bad(const char *why)
{
    std::snprintf(g_last_error, sizeof g_last_error, "invalid argument: %s", why);
    return MXQ_ERR_INVALID_ARG;
}

// Shape checks common to every entry point (pure host logic, no CUDA calls).
mxq_status check_shape(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0) return bad("negative size");
    if (cols % 32) return bad("cols must be a multiple of 32");
    if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31)) return bad("rows/cols must be < 2^31");
    if (rows > 0 && cols > 0 && rows * (cols / 32) >= (int64_t(1) << 31) - 512)
        return bad("rows * cols / 32 must be < 2^31 - 512");
    return MXQ_OK;
}

// Encoded tensor maps of recent calls, per host thread.  A map is a pure function of
// what it is encoded from (its kind, base address, extents and box), so a call that
// repeats those reuses the encoded map instead of encoding it again: repeated calls on
// the same buffers then skip cuTensorMapEncodeTiled.  Eight slots, replaced in turn.
struct TmapKey {
    int kind;
    const void *p;
    int64_t a, b;
    uint32_t box;
    bool operator==(const TmapKey &o) const
    {
        return kind == o.kind && p == o.p && a == o.a && b == o.b && box == o.box;
    }
};
struct TmapSlot {
    alignas(64) CUtensorMap map;
    TmapKey key;
    bool used;
};
constexpr int kTmapSlots = 8;
thread_local TmapSlot g_tmaps[kTmapSlots];
thread_local int g_tmap_next = 0;

bool tmap_lookup(const TmapKey &key, CUtensorMap *map)
{
    for (int i = 0; i < kTmapSlots; ++i) {
        if (g_tmaps[i].used && g_tmaps[i].key == key) {
            *map = g_tmaps[i].map;
            return true;
        }
    }
    return false;
}

void tmap_store(const TmapKey &key, const CUtensorMap &map)
{
    TmapSlot &slot = g_tmaps[g_tmap_next];
    g_tmap_next = (g_tmap_next + 1) % kTmapSlots;
    slot.map = map;
    slot.key = key;
    slot.used = true;
}

enum TmapKind { kMapCodes = 1, kMapGroups, kMapBlocks, kMapOperand, kMapSf, kMapX };

mxq_status make_tmap_codes(CUtensorMap *map, void *codes, int64_t rows, int64_t cols)
{
    const TmapKey key{kMapCodes, codes, rows, cols, 0};
    if (tmap_lookup(key, map)) return MXQ_OK;
    const Driver &d = driver();
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols / 2), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols / 2)};
    // one epilogue warp's store: 32 rows x 32 bytes (the codes of a 64-column tile), 32-byte swizzle
    // (16-byte chunk c of row r staged at chunk c ^ ((r >> 2) & 1), so the staging stores are conflict free)
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = d.encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        note_cu(r, "cuTensorMapEncodeTiled(codes)");
        return MXQ_ERR_CUDA;
    }
    tmap_store(key, *map);
    return MXQ_OK;
}

// A bf16 [rows, cols] matrix viewed as [rows*cols/32, 32]: one 64-byte row per group.
mxq_status make_tmap_groups(CUtensorMap *map, const void *X, int64_t rows, int64_t cols, uint32_t box_rows = 256)
{
    const TmapKey key{kMapGroups, X, rows, cols, box_rows};
    if (tmap_lookup(key, map)) return MXQ_OK;
    const Driver &d = driver();
    cuuint64_t dims[2] = {32, static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(cols / 32)};
    cuuint64_t strides[1] = {64};
    cuuint32_t box[2] = {32, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = d.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        note_cu(r, "cuTensorMapEncodeTiled(groups)");
        return MXQ_ERR_CUDA;
    }
    tmap_store(key, *map);
    return MXQ_OK;
}

// A bf16 [rows, cols] matrix viewed as [rows*cols/blk, blk]: one row per rotation block
// (blk = 64 or 128), loaded in 128-byte K-atoms of 64 columns, 16384/blk rows per box
// (32 KB of X per stage).
mxq_status make_tmap_blocks(CUtensorMap *map, const void *X, int64_t rows, int64_t cols, int blk)
{
    const TmapKey key{kMapBlocks, X, rows, cols, static_cast<uint32_t>(blk)};
    if (tmap_lookup(key, map)) return MXQ_OK;
    const Driver &d = driver();
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(blk),
                          static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(cols / blk)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(blk) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(16384 / blk)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = d.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        note_cu(r, "cuTensorMapEncodeTiled(blocks)");
        return MXQ_ERR_CUDA;
    }
    tmap_store(key, *map);
    return MXQ_OK;
}

// MXFP4 codes [rows, K/2] bytes as a GEMM operand: boxes of 128 bytes (256 k) x box_rows
// rows, 128-byte swizzle, zero fill past the edges.
mxq_status make_tmap_operand(CUtensorMap *map, const void *codes, int64_t rows, int64_t K, uint32_t box_rows)
{
    const TmapKey key{kMapOperand, codes, rows, K, box_rows};
    if (tmap_lookup(key, map)) return MXQ_OK;
    const Driver &d = driver();
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = d.encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        note_cu(r, "cuTensorMapEncodeTiled(gemm operand)");
        return MXQ_ERR_CUDA;
    }
    tmap_store(key, *map);
    return MXQ_OK;
}

// Scale atoms [row blocks][cb_n] x 512 B viewed as uint32 [row blocks][cb_n * 128]:
// boxes of two atoms (256 words) x box_rows row blocks, no swizzle, zero fill past the edges.
mxq_status make_tmap_sf(CUtensorMap *map, const void *atoms, int64_t row_blocks, int64_t cb_n, uint32_t box_rows)
{
    const TmapKey key{kMapSf, atoms, row_blocks, cb_n, box_rows};
    if (tmap_lookup(key, map)) return MXQ_OK;
    const Driver &d = driver();
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cb_n * 128), static_cast<cuuint64_t>(row_blocks)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cb_n * 512)};
    cuuint32_t box[2] = {256, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = d.encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(atoms), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        note_cu(r, "cuTensorMapEncodeTiled(scale atoms)");
        return MXQ_ERR_CUDA;
    }
    tmap_store(key, *map);
    return MXQ_OK;
}

mxq_status make_tmap_x(CUtensorMap *map, const void *X, int64_t rows, int64_t cols)
{
    const TmapKey key{kMapX, X, rows, cols, 0};
    if (tmap_lookup(key, map)) return MXQ_OK;
    const Driver &d = driver();
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(mxq::kTileM)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = d.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        note_cu(r, "cuTensorMapEncodeTiled");
        return MXQ_ERR_CUDA;
    }
    tmap_store(key, *map);
    return MXQ_OK;
}

// Common front half of the two rotate entry points.
// blk: the rotation block width (32 for the main path; 16, 64 or 128 for the variants).
mxq_status rotate_common(const void *X, int64_t rows, int64_t cols, const void *R, const float *lam,
                         void *out0, uint64_t out0_bytes, uint64_t out0_align, void *out1,
                         uint64_t out1_bytes, mxq::RotOut mode, void *stream, int blk = 32, int lam_mul = 0,
                         const float *nv_scale = nullptr)
{
    const bool quant = mode == mxq::RotOut::Quant || mxq::rot_nvfp4(mode) || mode == mxq::RotOut::QuantMma;
    const bool sf_mma = mxq::rot_sf_mma(mode);
    mxq_status st = check_shape(rows, cols);
    if (st != MXQ_OK) return st;
    if (blk != 16 && blk != 32 && blk != 64 && blk != 128) return bad("block must be 16, 32, 64 or 128");
    if (cols % blk) return bad("cols must be a multiple of the block width");
    if (lam && blk > 32) return bad("Lambda is supported with blocks of 16 or 32 columns only");
    if (rows == 0 || cols == 0) return MXQ_OK;   // nothing is read or written
    if (!X || !R || !out0 || (quant && !out1)) return bad("null pointer");
    if (mxq::rot_nvfp4(mode)) {
        if (blk != 32) return bad("NVFP4 takes a 32x32 Rhat");
        if (!nv_scale) return bad("null pointer");
        if (!aligned(nv_scale, 4)) return bad("tensor scale must be 4-byte aligned");
        if (!aligned(out1, 2)) return bad("NVFP4 scales must be 2-byte aligned");
    }
    if (sf_mma && !aligned(out1, 16)) return bad("MMA-layout scales must be 16-byte aligned");
    if (!aligned(X, 16)) return bad("X must be 16-byte aligned");
    if (!aligned(R, 2)) return bad("Rhat must be 2-byte aligned");
    if (lam && !aligned(lam, 4)) return bad("Lambda must be 4-byte aligned");
    if (!aligned(out0, out0_align)) return bad("output must be 16-byte aligned");
    const uint64_t nx = static_cast<uint64_t>(rows) * cols * 2, nl = lam ? static_cast<uint64_t>(cols) * 4 : 0;
    const uint64_t nr = static_cast<uint64_t>(blk) * blk * 2;
    const void *ins[4] = {X, R, lam, nv_scale};
    const uint64_t nins[4] = {nx, nr, nl, nv_scale ? 4u : 0u};
    for (int i = 0; i < 4; ++i) {
        if (overlaps(out0, out0_bytes, ins[i], nins[i]) || (out1 && overlaps(out1, out1_bytes, ins[i], nins[i])))
            return bad("an output overlaps an input");
    }
    if (out1 && overlaps(out0, out0_bytes, out1, out1_bytes)) return bad("outputs overlap");

    int dev = 0, sms = 0;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    if ((st = check_buffer(X, nx, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(R, nr, dev)) != MXQ_OK) return st;
    if (lam && (st = check_buffer(lam, nl, dev)) != MXQ_OK) return st;
    if (nv_scale && (st = check_buffer(nv_scale, 4, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(out0, out0_bytes, dev)) != MXQ_OK) return st;
    if (out1 && (st = check_buffer(out1, out1_bytes, dev)) != MXQ_OK) return st;

    alignas(64) CUtensorMap map_a;   // X as [n_groups, 32] (no smoothing), [n_blocks, blk] or [rows, cols]
    alignas(64) CUtensorMap map_c;   // the packed codes (smoothing, quantise mode)
    if (blk > 32) {
        if ((st = make_tmap_blocks(&map_a, X, rows, cols, blk)) != MXQ_OK) return st;
    } else if (lam == nullptr) {
        if ((st = make_tmap_groups(&map_a, X, rows, cols)) != MXQ_OK) return st;
    } else {
        if ((st = make_tmap_x(&map_a, X, rows, cols)) != MXQ_OK) return st;
        if (quant) {
            if ((st = make_tmap_codes(&map_c, out0, rows, cols)) != MXQ_OK) return st;
        } else {
            map_c = map_a;   // unused by the fp32 variant
        }
    }
    mxq::RotArgs args{};
    args.rhat = static_cast<const uint16_t *>(R);
    args.rblk = blk == 16 ? 16 : 32;
    args.lam_mul = lam_mul;
    args.nv_scale = nv_scale;
    args.lambda = lam;
    args.rows = rows;
    args.cols = cols;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (quant) {
        args.codes = static_cast<uint8_t *>(out0);
        if (sf_mma) {
            args.sf_mma = static_cast<uint8_t *>(out1);
            // the kernels write every scale of the matrix; the atoms' rows past it (rows not a
            // multiple of 128) and scale columns past it (cols/32 for MXFP4, cols/16 for NVFP4,
            // not a multiple of 4) must read 0
            const int64_t sc_cols = mode == mxq::RotOut::QuantNvMma ? cols / 16 : cols / 32;
            if (rows % 128 || sc_cols % 4) {
                const cudaError_t me = cudaMemsetAsync(out1, 0, out1_bytes, s);
                if (me != cudaSuccess) {
                    note_cuda(me, "cudaMemsetAsync(MMA-layout scales)");
                    return MXQ_ERR_CUDA;
                }
            }
        } else {
            args.scales = static_cast<uint8_t *>(out1);
        }
    } else {
        args.y = static_cast<float *>(out0);
    }
    cudaError_t e = blk > 32           ? mxq::launch_rotate_block(map_a, args, blk, mode, sms, s)
                    : lam == nullptr ? mxq::launch_rotate_flat(map_a, args, mode, sms, s)
                                     : mxq::launch_rotate_cols(map_a, map_c, args, mode, sms, s);
    if (e != cudaSuccess) {
        note_cuda(e, "launch rotate kernel");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

}  // namespace

namespace mxq {
void set_last_error(const char *msg) { std::snprintf(g_last_error, sizeof g_last_error, "%s", msg); }
}  // namespace mxq

extern "C" {

mxq_status mxq_smooth_rotate_quantize(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                                      const float *Lambda_or_null, uint8_t *out_codes_u8_packed,
                                      uint8_t *out_scales_e8m0, void *stream)
{
    const uint64_t nc = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols / 2 : 0;
    const uint64_t ns = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * (cols / 32) : 0;
    return rotate_common(X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_codes_u8_packed, nc, 16,
                         out_scales_e8m0, ns, mxq::RotOut::Quant, stream);
}

mxq_status mxq_smooth_rotate_quantize_mma(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                                          const float *Lambda_or_null, uint8_t *out_codes_u8_packed,
                                          uint8_t *out_scales_mma, void *stream)
{
    const uint64_t nc = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols / 2 : 0;
    const uint64_t ns = rows > 0 && cols > 0 && cols % 32 == 0 ? mxq_scales_mma_bytes(rows, cols) : 0;
    return rotate_common(X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_codes_u8_packed, nc, 16,
                         out_scales_mma, ns, mxq::RotOut::QuantMma, stream);
}

mxq_status mxq_smooth_rotate_quantize_nvfp4_mma(const void *X_bf16, int64_t rows, int64_t cols,
                                                const void *Rhat_bf16, const float *Lambda_or_null,
                                                const float *tensor_scale_f32, uint8_t *out_codes_u8_packed,
                                                uint8_t *out_scales_mma, void *stream)
{
    const uint64_t nc = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols / 2 : 0;
    const uint64_t ns = rows > 0 && cols > 0 && cols % 32 == 0 ? mxq_nvfp4_scales_mma_bytes(rows, cols) : 0;
    return rotate_common(X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_codes_u8_packed, nc, 16,
                         out_scales_mma, ns, mxq::RotOut::QuantNvMma, stream, 32, 0, tensor_scale_f32);
}

mxq_status mxq_smooth_rotate_f32(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                                 const float *Lambda_or_null, float *out_f32, void *stream)
{
    const uint64_t ny = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols * 4 : 0;
    return rotate_common(X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_f32, ny, 16, nullptr, 0,
                         mxq::RotOut::F32, stream);
}

mxq_status mxq_rotate_quantize_block(const void *X_bf16, int64_t rows, int64_t cols, int block, const void *R_bf16,
                                     const float *Lambda_or_null, uint8_t *out_codes_u8_packed,
                                     uint8_t *out_scales_e8m0, void *stream)
{
    const uint64_t nc = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols / 2 : 0;
    const uint64_t ns = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * (cols / 32) : 0;
    return rotate_common(X_bf16, rows, cols, R_bf16, Lambda_or_null, out_codes_u8_packed, nc, 16, out_scales_e8m0,
                         ns, mxq::RotOut::Quant, stream, block);
}

mxq_status mxq_rotate_block_f32(const void *X_bf16, int64_t rows, int64_t cols, int block, const void *R_bf16,
                                const float *Lambda_or_null, float *out_f32, void *stream)
{
    const uint64_t ny = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols * 4 : 0;
    return rotate_common(X_bf16, rows, cols, R_bf16, Lambda_or_null, out_f32, ny, 16, nullptr, 0,
                         mxq::RotOut::F32, stream, block);
}

mxq_status mxq_weight_rotate_quantize(const void *Wt_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                                      const float *Lambda_or_null, uint8_t *out_codes_u8_packed,
                                      uint8_t *out_scales_e8m0, void *stream)
{
    const uint64_t nc = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols / 2 : 0;
    const uint64_t ns = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * (cols / 32) : 0;
    return rotate_common(Wt_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_codes_u8_packed, nc, 16,
                         out_scales_e8m0, ns, mxq::RotOut::Quant, stream, 32, 1);
}

mxq_status mxq_smooth_rotate_quantize_nvfp4(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                                             const float *Lambda_or_null, const float *tensor_scale_f32,
                                             uint8_t *out_codes_u8_packed, uint8_t *out_scales_e4m3, void *stream)
{
    const uint64_t nc = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * cols / 2 : 0;
    const uint64_t ns = rows > 0 && cols > 0 ? static_cast<uint64_t>(rows) * (cols / 16) : 0;
    return rotate_common(X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_codes_u8_packed, nc, 16,
                         out_scales_e4m3, ns, mxq::RotOut::QuantNv, stream, 32, 0, tensor_scale_f32);
}

size_t mxq_scales_mma_bytes(int64_t rows, int64_t K)
{
    if (rows <= 0 || K <= 0 || K % 32) return 0;
    return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((K / 32 + 3) / 4) * 512;
}

mxq_status mxq_scales_to_mma_layout(const uint8_t *scales, int64_t rows, int64_t K, uint8_t *out, void *stream)
{
    if (rows < 0 || K < 0 || K % 32) return bad("rows >= 0 and K a multiple of 32 required");
    if (rows >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return bad("rows and K must be < 2^31");
    if (rows == 0 || K == 0) return MXQ_OK;
    if (!scales || !out) return bad("null pointer");
    if (!aligned(out, 16)) return bad("out must be 16-byte aligned");
    const uint64_t ns = static_cast<uint64_t>(rows) * (K / 32), no = mxq_scales_mma_bytes(rows, K);
    if (overlaps(out, no, scales, ns)) return bad("the output overlaps the input");
    int dev = 0, sms = 0;
    mxq_status st;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    if ((st = check_buffer(scales, ns, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(out, no, dev)) != MXQ_OK) return st;
    const cudaError_t e = mxq::launch_scales_to_mma(scales, rows, K / 32, out, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        note_cuda(e, "launch scale layout kernel");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

// MXFP4 (nv = 0) or NVFP4 (nv = 1, with the tensor scales) GEMM: validation and launch.
static mxq_status gemm_common(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *b_codes,
                              const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, void *out, int out_bf16,
                              void *stream, int nv, const float *a_tscale, const float *b_tscale)
{
    if (M < 0 || N < 0 || K < 0) return bad("negative size");
    if (K % 32) return bad("K must be a multiple of 32");
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return bad("M, N and K must be < 2^31");
    if (out_bf16 != 0 && out_bf16 != 1) return bad("out_bf16 must be 0 (fp32) or 1 (bf16)");
    if (M == 0 || N == 0) return MXQ_OK;
    const uint64_t ny = static_cast<uint64_t>(M) * N * (out_bf16 ? 2 : 4);
    if (!out) return bad("null pointer");
    if (!aligned(out, 16)) return bad("out must be 16-byte aligned");
    int dev = 0, sms = 0;
    mxq_status st = MXQ_OK;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (K == 0) {   // an empty sum: Y = 0
        if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
        if ((st = check_buffer(out, ny, dev)) != MXQ_OK) return st;
        const cudaError_t e = cudaMemsetAsync(out, 0, ny, s);
        if (e != cudaSuccess) {
            note_cuda(e, "cudaMemsetAsync");
            return MXQ_ERR_CUDA;
        }
        return MXQ_OK;
    }
    if (!a_codes || !a_scales || !b_codes || !b_scales) return bad("null pointer");
    if (nv && (!a_tscale || !b_tscale)) return bad("null pointer");
    if (!aligned(a_codes, 16) || !aligned(b_codes, 16)) return bad("codes must be 16-byte aligned");
    if (!aligned(a_scales, 16) || !aligned(b_scales, 16)) return bad("scale atoms must be 16-byte aligned");
    if (nv && (!aligned(a_tscale, 4) || !aligned(b_tscale, 4))) return bad("tensor scales must be 4-byte aligned");
    const uint64_t nca = static_cast<uint64_t>(M) * (K / 2), ncb = static_cast<uint64_t>(N) * (K / 2);
    const uint64_t nsa = nv ? mxq_nvfp4_scales_mma_bytes(M, K) : mxq_scales_mma_bytes(M, K);
    const uint64_t nsb = nv ? mxq_nvfp4_scales_mma_bytes(N, K) : mxq_scales_mma_bytes(N, K);
    const void *ins[6] = {a_codes, a_scales, b_codes, b_scales, a_tscale, b_tscale};
    const uint64_t nins[6] = {nca, nsa, ncb, nsb, nv ? 4u : 0u, nv ? 4u : 0u};
    for (int i = 0; i < 6; ++i)
        if (ins[i] && overlaps(out, ny, ins[i], nins[i])) return bad("the output overlaps an input");
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    for (int i = 0; i < 6; ++i)
        if (ins[i] && nins[i] && (st = check_buffer(ins[i], nins[i], dev)) != MXQ_OK) return st;
    if ((st = check_buffer(out, ny, dev)) != MXQ_OK) return st;
    alignas(64) CUtensorMap map_a, map_b, map_sfa, map_sfb;
    if ((st = make_tmap_operand(&map_a, a_codes, M, K, 128)) != MXQ_OK) return st;
    if ((st = make_tmap_operand(&map_b, b_codes, N, K, 128)) != MXQ_OK) return st;   // a CTA's half of B
    // scale atoms per 128-row block: one per 128 k (MXFP4) or per 64 k (NVFP4)
    const int64_t cb_n = nv ? (K / 16 + 3) / 4 : (K / 32 + 3) / 4;
    if ((st = make_tmap_sf(&map_sfa, a_scales, (M + 127) / 128, cb_n, 1)) != MXQ_OK) return st;
    if ((st = make_tmap_sf(&map_sfb, b_scales, (N + 127) / 128, cb_n, 2)) != MXQ_OK) return st;
    mxq::GemmArgs g{};
    g.y = out;
    g.M = M;
    g.N = N;
    g.K = K;
    g.out_bf16 = out_bf16;
    g.nvfp4 = nv;
    g.a_tscale = a_tscale;
    g.b_tscale = b_tscale;
    const cudaError_t e = mxq::launch_mxfp4_gemm(map_a, map_b, map_sfa, map_sfb, g, sms, s);
    if (e != cudaSuccess) {
        note_cuda(e, nv ? "launch NVFP4 GEMM kernel" : "launch MXFP4 GEMM kernel");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

mxq_status mxq_mxfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales_mma, const uint8_t *b_codes,
                          const uint8_t *b_scales_mma, int64_t M, int64_t N, int64_t K, void *out, int out_bf16,
                          void *stream)
{
    return gemm_common(a_codes, a_scales_mma, b_codes, b_scales_mma, M, N, K, out, out_bf16, stream, 0, nullptr,
                       nullptr);
}

size_t mxq_nvfp4_scales_mma_bytes(int64_t rows, int64_t K)
{
    if (rows <= 0 || K <= 0 || K % 32) return 0;
    return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((K / 16 + 3) / 4) * 512;
}

mxq_status mxq_nvfp4_scales_to_mma_layout(const uint8_t *scales, int64_t rows, int64_t K, uint8_t *out, void *stream)
{
    if (rows < 0 || K < 0 || K % 32) return bad("rows >= 0 and K a multiple of 32 required");
    if (rows >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return bad("rows and K must be < 2^31");
    if (rows == 0 || K == 0) return MXQ_OK;
    if (!scales || !out) return bad("null pointer");
    if (!aligned(out, 16)) return bad("out must be 16-byte aligned");
    const uint64_t ns = static_cast<uint64_t>(rows) * (K / 16), no = mxq_nvfp4_scales_mma_bytes(rows, K);
    if (overlaps(out, no, scales, ns)) return bad("the output overlaps the input");
    int dev = 0, sms = 0;
    mxq_status st;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    if ((st = check_buffer(scales, ns, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(out, no, dev)) != MXQ_OK) return st;
    // the same 512-byte atoms, four scale columns each: here a column is 16 k
    const cudaError_t e = mxq::launch_scales_to_mma(scales, rows, K / 16, out, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        note_cuda(e, "launch scale layout kernel");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

mxq_status mxq_nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales_mma, const float *a_tensor_scale,
                          const uint8_t *b_codes, const uint8_t *b_scales_mma, const float *b_tensor_scale, int64_t M,
                          int64_t N, int64_t K, void *out, int out_bf16, void *stream)
{
    return gemm_common(a_codes, a_scales_mma, b_codes, b_scales_mma, M, N, K, out, out_bf16, stream, 1,
                       a_tensor_scale, b_tensor_scale);
}

mxq_status mxq_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                          const void *Rhat_bf16_or_null, const float *Lambda_or_null, void *out_bf16,
                          void *stream)
{
    mxq_status st = check_shape(rows, cols);
    if (st != MXQ_OK) return st;
    if (rows == 0 || cols == 0) return MXQ_OK;   // nothing is read or written
    if (!codes || !scales || !out_bf16) return bad("null pointer");
    if (Lambda_or_null && !Rhat_bf16_or_null) return bad("Lambda requires Rhat");
    if (!aligned(codes, 16) || !aligned(out_bf16, 16)) return bad("codes and output must be 16-byte aligned");
    if (Rhat_bf16_or_null && !aligned(Rhat_bf16_or_null, 16)) return bad("Rhat must be 16-byte aligned for dequantize");
    if (Lambda_or_null && !aligned(Lambda_or_null, 4)) return bad("Lambda must be 4-byte aligned");
    const uint64_t nc = static_cast<uint64_t>(rows) * cols / 2, ns = static_cast<uint64_t>(rows) * (cols / 32);
    const uint64_t no = static_cast<uint64_t>(rows) * cols * 2;
    const uint64_t nl = Lambda_or_null ? static_cast<uint64_t>(cols) * 4 : 0;
    const uint64_t nr = Rhat_bf16_or_null ? 32 * 32 * 2 : 0;
    if (overlaps(out_bf16, no, codes, nc) || overlaps(out_bf16, no, scales, ns) ||
        overlaps(out_bf16, no, Rhat_bf16_or_null, nr) || overlaps(out_bf16, no, Lambda_or_null, nl))
        return bad("the output overlaps an input");
    int dev = 0, sms = 0;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    if ((st = check_buffer(codes, nc, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(scales, ns, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(out_bf16, no, dev)) != MXQ_OK) return st;
    if (Rhat_bf16_or_null && (st = check_buffer(Rhat_bf16_or_null, nr, dev)) != MXQ_OK) return st;
    if (Lambda_or_null && (st = check_buffer(Lambda_or_null, nl, dev)) != MXQ_OK) return st;
    cudaError_t e;
    if (Rhat_bf16_or_null) {
        alignas(64) CUtensorMap map_out;
        if ((st = make_tmap_groups(&map_out, out_bf16, rows, cols, 32)) != MXQ_OK) return st;
        e = mxq::launch_dequant_rot(map_out, codes, scales, rows, cols,
                                    static_cast<const uint16_t *>(Rhat_bf16_or_null), Lambda_or_null, sms,
                                    static_cast<cudaStream_t>(stream));
    } else {
        e = mxq::launch_dequant_plain(codes, scales, rows, cols, static_cast<uint16_t *>(out_bf16), sms,
                                      static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) {
        note_cuda(e, "launch dequantize kernel");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

size_t mxq_quant_error_workspace_bytes(int64_t rows, int64_t cols, int with_lambda)
{
    if (check_shape(rows, cols) != MXQ_OK || rows == 0 || cols == 0) return 0;
    const int64_t n = with_lambda ? mxq::rotate_cols_partials(rows, cols) : mxq::rotate_flat_partials(rows, cols);
    return static_cast<size_t>(n) * sizeof(double);
}

mxq_status mxq_quant_error(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                           const float *Lambda_or_null, float *out_group_err_or_null, double *out_mean,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    mxq_status st = check_shape(rows, cols);
    if (st != MXQ_OK) return st;
    if (!out_mean || !aligned(out_mean, 8)) return bad("out_mean must be an 8-byte aligned device double");
    if (rows == 0 || cols == 0) return bad("the mean of an empty matrix is undefined");
    if (!X_bf16 || !Rhat_bf16) return bad("null pointer");
    if (!aligned(X_bf16, 16)) return bad("X must be 16-byte aligned");
    if (!aligned(Rhat_bf16, 2)) return bad("Rhat must be 2-byte aligned");
    if (Lambda_or_null && !aligned(Lambda_or_null, 4)) return bad("Lambda must be 4-byte aligned");
    if (out_group_err_or_null && !aligned(out_group_err_or_null, 4))
        return bad("per-group errors must be 4-byte aligned");
    const size_t need = mxq_quant_error_workspace_bytes(rows, cols, Lambda_or_null != nullptr);
    if (!workspace || !aligned(workspace, 8) || workspace_bytes < need)
        return bad("workspace missing, not 8-byte aligned or smaller than mxq_quant_error_workspace_bytes()");
    const uint64_t nx = static_cast<uint64_t>(rows) * cols * 2;
    const uint64_t nl = Lambda_or_null ? static_cast<uint64_t>(cols) * 4 : 0;
    const uint64_t ne = out_group_err_or_null ? static_cast<uint64_t>(rows) * (cols / 32) * 4 : 0;
    const void *ins[3] = {X_bf16, Rhat_bf16, Lambda_or_null};
    const uint64_t nins[3] = {nx, 32 * 32 * 2, nl};
    void *outs[3] = {out_group_err_or_null, out_mean, workspace};
    const uint64_t nouts[3] = {ne, 8, need};
    for (int o = 0; o < 3; ++o) {
        for (int i = 0; i < 3; ++i)
            if (overlaps(outs[o], nouts[o], ins[i], nins[i])) return bad("an output overlaps an input");
        for (int o2 = o + 1; o2 < 3; ++o2)
            if (overlaps(outs[o], nouts[o], outs[o2], nouts[o2])) return bad("outputs overlap");
    }
    int dev = 0, sms = 0;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    if ((st = check_buffer(X_bf16, nx, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(Rhat_bf16, 32 * 32 * 2, dev)) != MXQ_OK) return st;
    if (Lambda_or_null && (st = check_buffer(Lambda_or_null, nl, dev)) != MXQ_OK) return st;
    if (out_group_err_or_null && (st = check_buffer(out_group_err_or_null, ne, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(out_mean, 8, dev)) != MXQ_OK) return st;
    if ((st = check_buffer(workspace, need, dev)) != MXQ_OK) return st;

    mxq::RotArgs args{};
    args.rhat = static_cast<const uint16_t *>(Rhat_bf16);
    args.lambda = Lambda_or_null;
    args.rows = rows;
    args.cols = cols;
    args.err = out_group_err_or_null;
    args.partials = static_cast<double *>(workspace);
    alignas(64) CUtensorMap map_a;
    cudaError_t e;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (Lambda_or_null == nullptr) {
        if ((st = make_tmap_groups(&map_a, X_bf16, rows, cols)) != MXQ_OK) return st;
        e = mxq::launch_rotate_flat(map_a, args, mxq::RotOut::Err, sms, s);
    } else {
        if ((st = make_tmap_x(&map_a, X_bf16, rows, cols)) != MXQ_OK) return st;
        e = mxq::launch_rotate_cols(map_a, map_a, args, mxq::RotOut::Err, sms, s);
    }
    if (e == cudaSuccess)
        e = mxq::launch_error_mean(args.partials, static_cast<int64_t>(need / sizeof(double)), rows * (cols / 32),
                                   out_mean, s);
    if (e != cudaSuccess) {
        note_cuda(e, "launch quantisation-error kernels");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

size_t mxq_rotation_search_workspace_bytes(int64_t rows, int64_t cols, int n_angle)
{
    if (check_shape(rows, cols) != MXQ_OK || rows < 1 || cols < 32 || n_angle < 1 || n_angle > 128) return 0;
    return mxq::rotation_search_workspace(rows, cols, n_angle);
}

mxq_status mxq_rotation_search(const void *X_bf16, int64_t rows, int64_t cols, const float *Lambda_or_null,
                               int max_steps, int n_angle, double *R_out, void *Rhat_bf16_out_or_null,
                               int32_t *trace_out_or_null, double *linf_out_or_null, int32_t *steps_out_or_null,
                               int64_t *group_out_or_null, void *workspace, size_t workspace_bytes, void *stream)
{
    mxq_status st = check_shape(rows, cols);
    if (st != MXQ_OK) return st;
    if (rows < 1 || cols < 32) return bad("the search needs at least one row and one group");
    if (max_steps < 0 || max_steps > 65536) return bad("max_steps must be in 0..65536");
    if (n_angle < 1 || n_angle > 128) return bad("n_angle must be in 1..128");
    if (!X_bf16 || !R_out) return bad("null pointer");
    if (!aligned(X_bf16, 16)) return bad("X must be 16-byte aligned");
    if (Lambda_or_null && !aligned(Lambda_or_null, 4)) return bad("Lambda must be 4-byte aligned");
    if (!aligned(R_out, 8)) return bad("R_out must be 8-byte aligned");
    if (Rhat_bf16_out_or_null && !aligned(Rhat_bf16_out_or_null, 2)) return bad("Rhat_out must be 2-byte aligned");
    if (trace_out_or_null && !aligned(trace_out_or_null, 4)) return bad("trace must be 4-byte aligned");
    if (linf_out_or_null && !aligned(linf_out_or_null, 8)) return bad("linf must be 8-byte aligned");
    if (steps_out_or_null && !aligned(steps_out_or_null, 4)) return bad("steps_out must be 4-byte aligned");
    if (group_out_or_null && !aligned(group_out_or_null, 8)) return bad("group_out must be 8-byte aligned");
    const size_t need = mxq_rotation_search_workspace_bytes(rows, cols, n_angle);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need)
        return bad("workspace missing, not 256-byte aligned or smaller than mxq_rotation_search_workspace_bytes()");
    const uint64_t nx = static_cast<uint64_t>(rows) * cols * 2;
    const uint64_t nl = Lambda_or_null ? static_cast<uint64_t>(cols) * 4 : 0;
    const void *ins[2] = {X_bf16, Lambda_or_null};
    const uint64_t nins[2] = {nx, nl};
    void *outs[7] = {R_out, Rhat_bf16_out_or_null, trace_out_or_null, linf_out_or_null, steps_out_or_null,
                     group_out_or_null, workspace};
    const uint64_t nouts[7] = {32 * 32 * 8,
                               Rhat_bf16_out_or_null ? 32 * 32 * 2u : 0u,
                               trace_out_or_null ? static_cast<uint64_t>(max_steps) * 12 : 0u,
                               linf_out_or_null ? static_cast<uint64_t>(max_steps + 1) * 8 : 0u,
                               steps_out_or_null ? 4u : 0u,
                               group_out_or_null ? 8u : 0u,
                               need};
    for (int o = 0; o < 7; ++o) {
        for (int i = 0; i < 2; ++i)
            if (overlaps(outs[o], nouts[o], ins[i], nins[i])) return bad("an output overlaps an input");
        for (int o2 = o + 1; o2 < 7; ++o2)
            if (overlaps(outs[o], nouts[o], outs[o2], nouts[o2])) return bad("outputs overlap");
    }
    int dev = 0, sms = 0;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    if ((st = check_buffer(X_bf16, nx, dev)) != MXQ_OK) return st;
    if (Lambda_or_null && (st = check_buffer(Lambda_or_null, nl, dev)) != MXQ_OK) return st;
    for (int o = 0; o < 7; ++o)
        if (outs[o] && nouts[o] && (st = check_buffer(outs[o], nouts[o], dev)) != MXQ_OK) return st;

    mxq::SearchArgs a{};
    a.X = X_bf16;
    a.lambda = Lambda_or_null;
    a.rows = rows;
    a.cols = cols;
    a.max_steps = max_steps;
    a.n_angle = n_angle;
    a.R = R_out;
    a.rhat = static_cast<uint16_t *>(Rhat_bf16_out_or_null);
    a.trace = trace_out_or_null;
    a.linf = linf_out_or_null;
    a.steps = steps_out_or_null;
    a.group = group_out_or_null;
    a.workspace = workspace;
    const cudaError_t e = mxq::launch_rotation_search(a, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        note_cuda(e, "launch rotation-search kernels");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

mxq_status mxq_sync_check(void *stream)
{
    unsigned int status = 0;
    cudaError_t e = mxq::read_and_clear_status(&status, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        note_cuda(e, "mxq_sync_check");
        return MXQ_ERR_CUDA;
    }
    if (status & mxq::kStatusTimeout) {
        std::snprintf(g_last_error, sizeof g_last_error, "a kernel's bounded wait ran out");
        return MXQ_ERR_TIMEOUT;
    }
    return MXQ_OK;
}

mxq_status mxq_selftest_bounded_wait(uint32_t timeout_ms, int *result_device, void *stream)
{
    if (!result_device || !aligned(result_device, 4)) return bad("result must be a 4-byte aligned device int");
    if (timeout_ms == 0 || timeout_ms > 10000) return bad("timeout_ms must be in 1..10000");
    int dev = 0, sms = 0;
    mxq_status st = current_device(&dev, &sms);
    if (st != MXQ_OK) return st;
    if ((st = check_buffer(result_device, 4, dev)) != MXQ_OK) return st;
    cudaError_t e = mxq::launch_wait_selftest(static_cast<uint64_t>(timeout_ms) * 1000000ull, result_device,
                                              static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        note_cuda(e, "launch wait self-test");
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

const char *mxq_status_string(mxq_status status)
{
    switch (status) {
    case MXQ_OK: return "MXQ_OK";
    case MXQ_ERR_INVALID_ARG: return "MXQ_ERR_INVALID_ARG: argument rejected before launch";
    case MXQ_ERR_UNSUPPORTED: return "MXQ_ERR_UNSUPPORTED: device is not an sm_100 part";
    case MXQ_ERR_CUDA: return "MXQ_ERR_CUDA: a CUDA call or kernel launch failed";
    case MXQ_ERR_TIMEOUT: return "MXQ_ERR_TIMEOUT: a kernel's bounded wait ran out";
    }
    return "unknown mxq_status";
}

const char *mxq_last_cuda_error(void) { return g_last_error; }

int mxq_version(void) { return 1 * 10000 + 0 * 100 + 0; }

}  // extern "C"
