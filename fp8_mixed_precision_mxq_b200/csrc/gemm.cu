// gemm.cu -- block-scaled MX GEMM on the 5th-generation tensor cores (sm_100a).
//
//   Y[M, N] = bf16( sum_k deqA[m, k] * deqW[n, k] + bias[n] )
//
// with A the quantized activation and W the MXFP4 weight, both K-major with one
// E8M0 scale per 32 elements along K.  This is the native W4A4 / W4A8 linear of the
// blog "Quark Mixed-Precision Quantization for Wan2.2 Video Generation on AMD
// Instinct GPUs" (section "Quantization formats", "Kernel note"): W4A4 runs
// tcgen05.mma kind::mxf4 (both operands E2M1, K = 64 per instruction); W4A8 runs
// kind::mxf8f6f4 with A in E4M3 and the E2M1 weight expanded by TMA into the
// byte-padded shared-memory form (K = 32 per instruction).
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: A / W tiles (128-byte swizzle) and the scale-factor
//               atoms (contiguous 512-byte chunks, plain bulk copies) into a
//               4-stage shared-memory ring;
//   warp 1      MMA issuer: copies each stage's scale atoms into TMEM
//               (tcgen05.cp 32x128b.warpx4) and issues the block-scaled MMAs into
//               a TMEM accumulator; allocates / frees TMEM;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, + bias, -> bf16, staged
//               in swizzled shared memory and written with TMA stores.
// TMEM (512 columns): accumulator slot 0 = columns [0, 256), slot 1 = [224, 480),
// scale factors = [480, 504).  The two slots overlap in [224, 256); the epilogue
// drains that 32-column chunk first and signals it, so the next tile's MMAs can
// start while the rest of the previous accumulator is still being written out.
// Every wait is bounded; a wait that runs out records MXQ_ERR_TIMEOUT in a device
// status word and the kernel winds down (in-flight copies and MMAs drained, TMEM
// freed) instead of hanging.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>

#include "mxq_internal.h"
#include "ptx.cuh"

namespace mxq {

__device__ uint32_t g_device_status;

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int kStages = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kStageA = BM * 128;               // 128 rows x 128 bytes
constexpr uint32_t kStageB = BN * 128;               // 256 rows x 128 bytes
constexpr uint32_t kStageSFA = 2 * 512;              // up to two k-atoms
constexpr uint32_t kStageSFB = 2 * 2 * 512;          // two 128-row halves x two k-atoms
constexpr uint32_t kEpiBuf = 32 * 64;                // 32 rows x 32 bf16
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kStageA;
constexpr uint32_t kOffSFA = kOffB + kStages * kStageB;
constexpr uint32_t kOffSFB = kOffSFA + kStages * kStageSFA;
constexpr uint32_t kOffEpi = kOffSFB + kStages * kStageSFB;
constexpr uint32_t kOffBar = kOffEpi + kEpiWarps * 2 * kEpiBuf;
constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1 + 1;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol1 = 224;
constexpr uint32_t kSfaCol = 480;
constexpr uint32_t kSfbCol = 488;
constexpr int kGroupM = 16;  // m-blocks per rasterization group
constexpr uint64_t kWaitNs = 1000000000ull;

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffEpi % 1024 == 0 && kOffB % 1024 == 0, "swizzled buffers need 1024-byte alignment");

struct Params {
    const uint8_t* a_sf;
    const uint8_t* w_sf;
    const __nv_bfloat16* bias;
    int M, N, K;
    int m_blocks, n_blocks, num_tiles, k_stages, atoms_k, sf_rows_w;
    uint32_t debug;
};

__device__ __forceinline__ void record_timeout()
{
    atomicCAS(&g_device_status, 0u, static_cast<uint32_t>(MXQ_ERR_TIMEOUT));
}

__device__ __forceinline__ void tile_coords(int t, int m_blocks, int n_blocks, int& mb, int& nb)
{
    const int per_group = kGroupM * n_blocks;
    const int gid = t / per_group;
    const int first_m = gid * kGroupM;
    const int gsize = min(kGroupM, m_blocks - first_m);
    const int local = t - gid * per_group;
    nb = local / gsize;
    mb = first_m + (local - nb * gsize);
}

template <bool kW4A8>
__global__ void __launch_bounds__(kThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_y, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* tmem_full = bars + 2 * kStages;
    uint64_t* tmem_empty = bars + 2 * kStages + 2;
    uint64_t* overlap_free = bars + 2 * kStages + 4;
    uint64_t* mma_done = bars + 2 * kStages + 5;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // k-atoms (128 K-elements of scale factors) per pipeline stage
    constexpr int AK = kW4A8 ? 1 : 2;

    if (warp == 0 && lane == 0) {
        prefetch_tmap(&map_a);
        prefetch_tmap(&map_b);
        prefetch_tmap(&map_y);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tmem_full[s], 1);
            mbar_init(&tmem_empty[s], kEpiWarps);
        }
        mbar_init(overlap_free, kEpiWarps);
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;          // stages issued (including a skipped one)
            int64_t skipped = -1;     // debug: index of the stage whose load was skipped
            bool ok = true;
            const int n_row_tiles_w = p.sf_rows_w;
            for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p.m_blocks, p.n_blocks, mb, nb);
                for (int ks = 0; ks < p.k_stages; ++ks, ++it) {
                    const uint32_t s = it % kStages;
                    if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, kWaitNs)) {
                        record_timeout();
                        ok = false;
                        break;
                    }
                    if ((p.debug & 1u) && it == 0 && blockIdx.x == 0) {
                        skipped = 0;  // deliberately leave stage 0 unfilled
                        continue;
                    }
                    const int ka0 = ks * AK;
                    const int na = min(AK, p.atoms_k - ka0);
                    const int rt0 = nb * 2;
                    const int nh = min(2, n_row_tiles_w - rt0);
                    const uint32_t tx = kStageA + (kW4A8 ? kStageB / 2 : kStageB) + na * 512u * (1 + nh);
                    mbar_arrive_expect_tx(&full[s], tx);
                    tma_load_2d(smem + kOffA + s * kStageA, &map_a, ks * 128, mb * BM, &full[s]);
                    tma_load_2d(smem + kOffB + s * kStageB, &map_b, ks * 128, nb * BN, &full[s]);
                    bulk_load(smem + kOffSFA + s * kStageSFA,
                              p.a_sf + (static_cast<int64_t>(mb) * p.atoms_k + ka0) * 512, na * 512u, &full[s]);
                    for (int h = 0; h < nh; ++h)
                        bulk_load(smem + kOffSFB + s * kStageSFB + h * AK * 512,
                                  p.w_sf + (static_cast<int64_t>(rt0 + h) * p.atoms_k + ka0) * 512, na * 512u,
                                  &full[s]);
                }
            }
            // drain: every load still in flight lands before the CTA may exit
            const uint32_t first = it > kStages ? it - kStages : 0;
            for (uint32_t i = first; i < it; ++i) {
                if (static_cast<int64_t>(i) == skipped) continue;
                if (!mbar_wait(&full[i % kStages], (i / kStages) & 1, kWaitNs)) record_timeout();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t fa = kW4A8 ? 0u : 1u;   // A element type: E4M3 (mxf8f6f4) / E2M1 (mxf4)
            const uint32_t fb = kW4A8 ? 5u : 1u;   // B element type: E2M1 in both kinds
            uint32_t it = 0;
            int tcount = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++tcount) {
                const int slot = tcount & 1;
                const uint32_t acc = tmem_base + (slot ? kAccCol1 : 0u);
                if (!mbar_wait(&tmem_empty[slot], ((tcount >> 1) & 1) ^ 1, kWaitNs) ||
                    (tcount > 0 && !mbar_wait(overlap_free, (tcount - 1) & 1, kWaitNs))) {
                    record_timeout();
                    break;
                }
                tc_fence_after();
                int mb, nb;
                tile_coords(t, p.m_blocks, p.n_blocks, mb, nb);
                const int nh = min(2, p.sf_rows_w - nb * 2);
                for (int ks = 0; ks < p.k_stages; ++ks, ++it) {
                    const uint32_t s = it % kStages;
                    if (!mbar_wait(&full[s], (it / kStages) & 1, kWaitNs)) {
                        record_timeout();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int na = min(AK, p.atoms_k - ks * AK);
                    const uint32_t sfa_s = smem_u32(smem + kOffSFA + s * kStageSFA);
                    const uint32_t sfb_s = smem_u32(smem + kOffSFB + s * kStageSFB);
                    for (int a = 0; a < na; ++a) {
                        tc_copy_sf_atom(tmem_base + kSfaCol + 4 * a, sdesc_sf_atom(sfa_s + a * 512));
                        for (int h = 0; h < nh; ++h)
                            tc_copy_sf_atom(tmem_base + kSfbCol + 8 * a + 4 * h,
                                            sdesc_sf_atom(sfb_s + (h * AK + a) * 512));
                    }
                    const uint32_t a_s = smem_u32(smem + kOffA + s * kStageA);
                    const uint32_t b_s = smem_u32(smem + kOffB + s * kStageB);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int k_elem = kW4A8 ? ks * 128 + j * 32 : ks * 256 + j * 64;
                        if (k_elem >= p.K) break;
                        const int atom = kW4A8 ? 0 : (j >> 1);
                        const uint32_t sf_id = kW4A8 ? static_cast<uint32_t>(j) : static_cast<uint32_t>((j & 1) * 2);
                        const uint32_t idesc = idesc_block_scaled(fa, fb, BM, BN, sf_id, sf_id);
                        const uint64_t ad = sdesc_k_sw128(a_s + j * 32);
                        const uint64_t bd = sdesc_k_sw128(b_s + j * 32);
                        const uint32_t accumulate = (ks > 0 || j > 0) ? 1u : 0u;
                        if (kW4A8)
                            mma_mxf8f6f4(acc, ad, bd, idesc, tmem_base + kSfaCol + 4 * atom,
                                         tmem_base + kSfbCol + 8 * atom, accumulate);
                        else
                            mma_mxf4(acc, ad, bd, idesc, tmem_base + kSfaCol + 4 * atom,
                                     tmem_base + kSfbCol + 8 * atom, accumulate);
                    }
                    tc_commit(&empty[s]);  // stage s is free once these MMAs completed
                }
                if (!ok) break;
                tc_commit(&tmem_full[slot]);  // accumulator ready for the epilogue
            }
            // every MMA issued by this thread completes before TMEM is released
            tc_commit(mma_done);
            if (!mbar_wait(mma_done, 0, kWaitNs)) record_timeout();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        uint8_t* ebuf0 = smem + kOffEpi + ew * 2 * kEpiBuf;
        int eb = 0;
        int tcount = 0;
        for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++tcount) {
            const int slot = tcount & 1;
            if (!mbar_wait(&tmem_full[slot], (tcount >> 1) & 1, kWaitNs)) {
                record_timeout();
                break;
            }
            tc_fence_after();
            int mb, nb;
            tile_coords(t, p.m_blocks, p.n_blocks, mb, nb);
            const uint32_t col0 = slot ? kAccCol1 : 0u;
            const int row0 = mb * BM + q * 32;
            for (int ci = 0; ci < BN / 32; ++ci) {
                // the 32 columns shared by both slots go first
                const int c = slot ? ci : (ci == 0 ? BN / 32 - 1 : ci - 1);
                uint32_t r[32];
                tmem_ld_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + col0 + c * 32, r);
                tmem_ld_wait();
                if (ci == 0) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(overlap_free);
                }
                const int n = nb * BN + c * 32;
                if (n >= p.N) continue;
                float bv[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) bv[i] = 0.f;
                if (p.bias != nullptr) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        if (n + 8 * g + 8 <= p.N) {
                            const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.bias + n + 8 * g));
                            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                bv[8 * g + 2 * i] = __uint_as_float(w[i] << 16);
                                bv[8 * g + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
                            }
                        }
                    }
                }
                uint32_t o[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * i]) + bv[2 * i],
                                                             __uint_as_float(r[2 * i + 1]) + bv[2 * i + 1]);
                    o[i] = *reinterpret_cast<uint32_t*>(&h);
                }
                uint8_t* buf = ebuf0 + eb * kEpiBuf;
                if (lane == 0) bulk_wait_read<1>();  // the store that last used buf has read it
                __syncwarp();
                const uint32_t rsw = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint4* dst = reinterpret_cast<uint4*>(buf + lane * 64 + ((ch ^ rsw) * 16));
                    *dst = make_uint4(o[4 * ch], o[4 * ch + 1], o[4 * ch + 2], o[4 * ch + 3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&map_y, buf, n, row0);
                    bulk_commit();
                }
                eb ^= 1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[slot]);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------- host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                 uint64_t stride_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint32_t g_debug_flags = 0;

}  // namespace

void set_debug_flags(uint32_t flags) { g_debug_flags = flags; }
uint32_t debug_flags() { return g_debug_flags; }

int read_and_clear_device_status(cudaStream_t stream, uint32_t* out)
{
    uint32_t v = 0, zero = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MXQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return MXQ_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero) != cudaSuccess) return MXQ_ERR_CUDA;
    *out = v;
    return MXQ_OK;
}

int launch_gemm(const GemmArgs& g, cudaStream_t stream, const char** msg, char* path, size_t path_len)
{
    const bool w4a8 = g.a_fmt == kFmtE4M3;
    CUtensorMap ma, mb, my;
    const uint64_t a_row = w4a8 ? g.K : g.K / 2;
    bool ok = make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a_codes, a_row, g.M, a_row, 128, BM,
                          CU_TENSOR_MAP_SWIZZLE_128B);
    if (w4a8)
        ok = ok && make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, g.w_codes, g.K, g.N, g.K / 2, 128, BN,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    else
        ok = ok && make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w_codes, g.K / 2, g.N, g.K / 2, 128, BN,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.y, g.N, g.M, g.N * 2, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_64B);
    if (!ok) {
        *msg = "cuTensorMapEncodeTiled failed (driver entry point unavailable or invalid operand layout)";
        return MXQ_ERR_CUDA;
    }
    Params p;
    p.a_sf = static_cast<const uint8_t*>(g.a_sf);
    p.w_sf = static_cast<const uint8_t*>(g.w_sf);
    p.bias = static_cast<const __nv_bfloat16*>(g.bias);
    p.M = static_cast<int>(g.M);
    p.N = static_cast<int>(g.N);
    p.K = static_cast<int>(g.K);
    p.m_blocks = static_cast<int>(ceil_div(g.M, BM));
    p.n_blocks = static_cast<int>(ceil_div(g.N, BN));
    p.num_tiles = p.m_blocks * p.n_blocks;
    p.k_stages = static_cast<int>(ceil_div(g.K, w4a8 ? 128 : 256));
    p.atoms_k = static_cast<int>(sf_atoms_k(g.K));
    p.sf_rows_w = static_cast<int>(ceil_div(g.N, 128));
    p.debug = g_debug_flags;

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(p.num_tiles, sms);
    cudaError_t e;
    if (w4a8) {
        e = cudaFuncSetAttribute(mx_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e == cudaSuccess) mx_gemm_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(ma, mb, my, p);
    } else {
        e = cudaFuncSetAttribute(mx_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e == cudaSuccess) mx_gemm_kernel<false><<<grid, kThreads, kSmemBytes, stream>>>(ma, mb, my, p);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        *msg = cudaGetErrorString(e);
        return MXQ_ERR_CUDA;
    }
    if (path)
        snprintf(path, path_len, "native %s 1cta %dx%d grid %d tiles %d", w4a8 ? "mxf8f6f4" : "mxf4", BM, BN, grid,
                 p.num_tiles);
    return MXQ_OK;
}

}  // namespace mxq
