// prepare.cu -- the forward's operand preparation for sm_100a: Q and K to
// MXFP4 rows and V to MXFP4 V^T, with every scale group in the regrouped
// order the attention kernel's tcgen05.cp reads, in one persistent launch.
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
// Quantization for MXFP4 Attention", abstract -- MXFP4 operands with
// power-of-two microscaling; scale rule OCP (floor(log2 amax) - 2) or UOS
// (smallest e with amax <= Qmax * 2^e, Qmax = 7.25).  The arithmetic per block
// is shared with the standalone quantizers (quantize_quad_bf16 and
// quantize_vt_block_bf16 in mxfp4_block.cuh).
//
// The work is a list of tiles of 128 tokens x d channels of bf16 (32 KB for
// d = 128): for every (b, h) and 128-token group, its Q, K and V tile, in that
// order, so the heavier V^T tiles spread evenly over the CTAs.  Each CTA (three
// per SM) takes every gridDim.x-th tile:
//   * one producer lane streams the tiles into a two-slot shared-memory ring
//     with TMA (rows past N arrive as zeros);
//   * 2 d consumer threads quantize the tile in the ring slot while the next
//     tiles are in flight:
//       Q / K tile: a quad of lanes per 32-channel block, 16-byte shared loads,
//         one 32-bit code store per lane, the quad's scale byte stored straight
//         into the regrouped group;
//       V tile: a thread per (channel pair, 32-token run), one 32-bit shared
//         read per token for both channels, 16-byte code stores per channel,
//         its two scale bytes stored straight into the regrouped group.
// 2.53125 bytes per element (2 read, 0.5 codes, 1/32 scale).  The consumers'
// arithmetic, not the bytes in flight, sets the pace: on the video-DiT inputs
// (1.27 GB) one CTA per SM with four slots takes 0.321 ms, two CTAs with three
// slots 0.240 ms, three CTAs with two slots 0.234 ms (the two separate
// kernels this replaces took 0.247 ms).
// No consumer waits on another (no named barrier), so a wait that gives up in
// one warp cannot leave the others blocked.  Every mbarrier wait is bounded; a
// wait that gives up records MXATTN_ERR_TIMEOUT in the status word, and the
// producer waits for its own copies in flight before the CTA exits.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "kernels.cuh"
#include "mxfp4_block.cuh"
#include "ptx.cuh"

namespace mxattn {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

namespace {

constexpr uint64_t kPrepTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kPrepTimeoutCode = 4u;           // MXATTN_ERR_TIMEOUT
// Ring slots per CTA and CTAs per SM (measured best: two slots, three CTAs).
#ifndef MXATTN_PREP_STAGES
#define MXATTN_PREP_STAGES 2
#endif
#ifndef MXATTN_PREP_CTAS
#define MXATTN_PREP_CTAS 3
#endif

template <int D>
struct PrepCfg {
    static constexpr int kStages = MXATTN_PREP_STAGES;
    static constexpr int kTileBytes = 128 * D * 2;
    static constexpr int kConsumers = 2 * D;             // 256 (d = 128) or 128 (d = 64)
    static constexpr int kThreads = kConsumers + 32;     // + the producer warp
    static constexpr int kChunksPerRow = D / 8;          // 16-byte chunks of a bf16 row
    static constexpr int kChunksPerThread = 128 * kChunksPerRow / kConsumers;  // Q / K: 8
    static constexpr int kPairs = D / 2;                 // V: channel pairs
    static constexpr int kRuns = kConsumers / kPairs;    // V: 32-token runs per tile (4)
    static_assert(kRuns * 32 == 128, "one 32-token block per V thread");
    // shared memory: the ring, barriers, flags
    static constexpr int kOffBar = kStages * kTileBytes;
    static constexpr int kOffMisc = kOffBar + 2 * kStages * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
};

struct PrepArgs {
    uint8_t* q_codes;   // [BH, N, d/2]
    uint8_t* k_codes;
    uint8_t* vt_codes;  // [BH, d, Npad/2]
    uint8_t* q_sf;      // regrouped [BH, G, 512]
    uint8_t* k_sf;
    uint8_t* v_sf;
    uint32_t* status;
    int N;
    int npad;
    int groups;
    int64_t n_tiles;  // 3 * BH * groups
    uint32_t sf_thresh;
};

template <int D>
__global__ void __launch_bounds__(PrepCfg<D>::kThreads, MXATTN_PREP_CTAS)
    prepare_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrepArgs p) {
    using C = PrepCfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = smem;
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_empty = bar_full + S;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
    volatile int* no_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);  // stays 0
    const int tid = threadIdx.x;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bar_full + s, 1);
            mbar_init(bar_empty + s, C::kConsumers);
        }
        *abort_flag = 0;
        *no_abort = 0;
        fence_mbarrier_init();
        if (blockIdx.x == 0) *p.status = 0u;
    }
    __syncthreads();

    if (tid >= C::kConsumers) {
        // ------------------------------------------------------------ TMA producer (one lane)
        const bool leader = elect_one_sync();
        int64_t issued = 0;
        for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++issued) {
            const int s = static_cast<int>(issued % S);
            const uint32_t n = static_cast<uint32_t>(issued / S);
            if (issued >= S &&
                !__all_sync(0xffffffffu, mbar_wait_bounded(bar_empty + s, (n - 1) & 1, abort_flag, p.status,
                                                            kPrepTimeoutCode, kPrepTimeoutNs)))
                break;
            if (leader) {
                const int z = static_cast<int>(tile % 3);  // Q, K, V
                const int64_t bg = tile / 3;               // bh * groups + g
                const int bh = static_cast<int>(bg / p.groups);
                const int g = static_cast<int>(bg % p.groups);
                mbar_arrive_expect_tx(bar_full + s, C::kTileBytes);
                tma_load_3d(ring + s * C::kTileBytes, z == 0 ? &tmQ : (z == 1 ? &tmK : &tmV), bar_full + s, 0,
                            g * 128, bh);
            }
            __syncwarp();
        }
        // Every copy issued must land before the CTA exits (on the normal path the
        // consumers have waited for all of them already).
        for (int64_t i = issued - S < 0 ? 0 : issued - S; i < issued; ++i)
            mbar_wait_bounded(bar_full + i % S, static_cast<uint32_t>(i / S) & 1, no_abort, p.status, kPrepTimeoutCode,
                              kPrepTimeoutNs);
        return;
    }

    // ---------------------------------------------------------------- consumers
    int64_t used = 0;
    for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++used) {
        const int s = static_cast<int>(used % S);
        const uint32_t n = static_cast<uint32_t>(used / S);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_full + s, n & 1, abort_flag, p.status, kPrepTimeoutCode,
                                                        kPrepTimeoutNs)))
            break;
        const int z = static_cast<int>(tile % 3);
        const int64_t bg = tile / 3;
        const int64_t bh = bg / p.groups;
        const int g = static_cast<int>(bg % p.groups);
        const uint8_t* t8 = ring + s * C::kTileBytes;
        const int t0 = g * 128;
        if (z < 2) {
            // Q / K rows: chunk c (8 channels) of row m; lanes 4k .. 4k + 3 hold one 32-channel block.
            uint8_t* grp = (z == 0 ? p.q_sf : p.k_sf) + bg * 512;
            uint32_t* codes = reinterpret_cast<uint32_t*>(z == 0 ? p.q_codes : p.k_codes);
            uint4 raw[C::kChunksPerThread];
#pragma unroll
            for (int u = 0; u < C::kChunksPerThread; ++u)
                raw[u] = reinterpret_cast<const uint4*>(t8)[tid + u * C::kConsumers];
            __syncwarp();
            mbar_arrive(bar_empty + s);  // the ring slot is free once its bytes are in registers
#pragma unroll
            for (int u = 0; u < C::kChunksPerThread; ++u) {
                const int c = tid + u * C::kConsumers;
                const int m = c / C::kChunksPerRow;
                const int cc = c % C::kChunksPerRow;
                int e;
                const uint32_t packed = quantize_quad_bf16(raw[u], p.sf_thresh, e);
                if (t0 + m < p.N) codes[(bh * p.N + t0 + m) * (D / 8) + cc] = packed;
                // row m's scale word: byte k for its block k (rows past N: zero data, byte 0)
                uint8_t* word = grp + (m & 31) * 16 + (m >> 5) * 4;
                if ((tid & 3) == 0) word[cc / 4] = static_cast<uint8_t>(e + 127);
                if (D == 64 && (tid & 7) == 0) *reinterpret_cast<uint16_t*>(word + 2) = 0;  // bytes of blocks 2, 3
            }
        } else {
            // V^T: thread = (channel pair cp, 32-token run); token i of the run's block holds
            // channel 2 cp in the low half of its 32-bit word and 2 cp + 1 in the high half.
            const int cp = tid % C::kPairs;
            const int run = tid / C::kPairs;
            const uint32_t* tile32 = reinterpret_cast<const uint32_t*>(t8);
            uint32_t raw[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) raw[i] = tile32[(run * 32 + i) * C::kPairs + cp];
            mbar_arrive(bar_empty + s);
            uint32_t words[2][4];
            int e[2];
            quantize_vt_block_bf16(raw, p.sf_thresh, words, e);
            const int tb = t0 + run * 32;  // first token of the block
            uint8_t* grp = p.v_sf + bg * 512;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int ch = 2 * cp + h;
                if (tb < p.npad)
                    *reinterpret_cast<uint4*>(p.vt_codes + (bh * D + ch) * static_cast<int64_t>(p.npad / 2) + tb / 2) =
                        make_uint4(words[h][0], words[h][1], words[h][2], words[h][3]);
                // channel ch plays the role of the row, block `run` of the group its byte
                grp[(ch & 31) * 16 + (ch >> 5) * 4 + run] = static_cast<uint8_t>(e[h] + 127);
            }
            if (D < 128 && run == 0) {
                // channel rows D..127 of the group: scale 2^0, so the extra ones-row the
                // attention kernel appends to V^T (row D) is read with unit scale
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c2 = 2 * cp + h + D;
                    *reinterpret_cast<uint32_t*>(grp + (c2 & 31) * 16 + (c2 >> 5) * 4) = 0x7F7F7F7Fu;
                }
            }
        }
    }
}

// 3-D bf16 tensor [BH, N, d] with a (d x 128 x 1) box, no swizzle.
bool encode_bf16_tiles(CUtensorMap* map, const void* base, int64_t BH, int N, int d) {
    auto fn = tensor_map_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(d) * 2 * N};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(d), 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_prepare_impl(const void* Q, const void* K, const void* V, int64_t BH, int N, uint32_t sf_thresh,
                                int groups, uint8_t* q_codes, uint8_t* k_codes, uint8_t* vt_codes, uint8_t* q_sf,
                                uint8_t* k_sf, uint8_t* v_sf, uint32_t* status, cudaStream_t stream) {
    using C = PrepCfg<D>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(prepare_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap tq, tk, tv;
    if (!encode_bf16_tiles(&tq, Q, BH, N, D) || !encode_bf16_tiles(&tk, K, BH, N, D) ||
        !encode_bf16_tiles(&tv, V, BH, N, D))
        return cudaErrorInvalidValue;
    PrepArgs a{};
    a.q_codes = q_codes;
    a.k_codes = k_codes;
    a.vt_codes = vt_codes;
    a.q_sf = q_sf;
    a.k_sf = k_sf;
    a.v_sf = v_sf;
    a.status = status;
    a.N = N;
    a.npad = (N + 31) / 32 * 32;
    a.groups = groups;
    a.n_tiles = 3 * BH * groups;
    a.sf_thresh = sf_thresh;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = a.n_tiles;
    const int grid = static_cast<int>(want < MXATTN_PREP_CTAS * sms ? want : MXATTN_PREP_CTAS * sms);
    prepare_kernel<D><<<grid, C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prepare(const void* Q, const void* K, const void* V, int64_t BH, int N, int d, uint32_t sf_thresh,
                           int groups, uint8_t* q_codes, uint8_t* k_codes, uint8_t* vt_codes, uint8_t* q_sf,
                           uint8_t* k_sf, uint8_t* v_sf, uint32_t* status, cudaStream_t stream) {
    if (d == 128)
        return launch_prepare_impl<128>(Q, K, V, BH, N, sf_thresh, groups, q_codes, k_codes, vt_codes, q_sf, k_sf,
                                        v_sf, status, stream);
    if (d == 64)
        return launch_prepare_impl<64>(Q, K, V, BH, N, sf_thresh, groups, q_codes, k_codes, vt_codes, q_sf, k_sf,
                                       v_sf, status, stream);
    return cudaErrorInvalidValue;
}

}  // namespace mxattn
