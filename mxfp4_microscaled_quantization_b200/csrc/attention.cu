// attention.cu -- fused MXFP4 attention forward with UOS and PNQ for sm_100a.
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
// Quantization for MXFP4 Attention", abstract: MXFP4 attention whose softmax
// loop quantizes the unnormalized exponentials exp(S - m) of each key tile to
// MXFP4 (scale rule UOS, Qmax = 7.25, or OCP) before the row sum, so the sum
// is built from the same quantized values that weight V (PNQ).
//
// One CTA owns two 128-row query tiles (A and B) of one (batch, head) and
// walks all key tiles in ascending order; both tiles share every K / V^T tile
// and one TMEM buffer for S, and their softmax warpgroups run a half-step
// apart (ping-pong), so one tile's serial phases (TMEM load, waits, O
// rescale, P hand-off) overlap the other tile's exponentials.  Roles (384
// threads, three warpgroups; setmaxnreg gives the two softmax warpgroups 224
// registers per thread and the third 56):
//   warps 0-3 / 4-7    softmax for tile A / B, one thread per query row (=
//                      TMEM lane): running max, per-32-column block exponent
//                      (UOS/OCP) in the log domain, the exponentials with the
//                      block scale folded into the bias of one FMA -- under
//                      PNQ 9 of 16 pairs on the MUFU and 7 on the FMA pipe (a
//                      code-only stand-in for 2^w; NVFP4 8 and 8), without
//                      PNQ 10 and 6 (a full polynomial exponential) -- E2M1
//                      packing of P into
//                      shared memory, O rescale in TMEM when the max moved,
//                      and the final O / l.
//   warp 8 (one lane)  TMA producer: both Q tiles + scales once, then K and
//                      V^T tiles (+ scales) into a kStages-deep ring.
//   warp 9 (one lane)  S issuer: tcgen05.cp of the Q and K scales into TMEM
//                      and S_A(j) = Q_A K(j)^T, S_B(j) = Q_B K(j)^T
//                      (tcgen05.mma kind::mxf4 block_scale) into the shared S
//                      buffer, each as soon as the other tile has read the
//                      buffer; it also allocates and frees TMEM.
//   warp 10 (one lane) PV issuer: tcgen05.cp of the P and V^T scales and
//                      O_A += P_A V(j), O_B += P_B V(j) as each P arrives.
//                      With the S and PV products on two issuing threads, a
//                      tile's next S never waits in program order behind the
//                      other tile's P.
//   warp 11            idle (it completes the third warpgroup).
// The row sum under PNQ is produced by the tensor core itself: V^T gets one
// extra row of ones (E2M1 1.0, scale 2^0) so O's column d accumulates
// sum_j q_j -- exactly the quantized values that multiply V -- and is
// rescaled together with O.  Without PNQ the row sum of the unquantized
// exponentials is kept in a register.
//
// The same template with NV = true is the NVFP4 comparison variant:
// tcgen05.mma kind::mxf4nvf4 block16 with E4M3 scale factors, P in blocks of
// 16 keys with E4M3 scales, and per-(batch, head) second-level scales folded
// into the softmax scale and the epilogue.
//
// Every mbarrier wait is bounded (kTimeoutNs); a wait that gives up records
// MXATTN_ERR_TIMEOUT in the status word, raises a CTA-wide abort flag, and
// every role drains its in-flight copies / MMAs before the CTA frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {

namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kTimeoutCode = 4u;           // MXATTN_ERR_TIMEOUT
#ifndef MXATTN_ROLE_WAIT_HINT_NS
#define MXATTN_ROLE_WAIT_HINT_NS 0
#endif
// Suspend hint for the producer's and the MMA issuer's waits (0: plain try_wait).
constexpr uint32_t kRoleWaitHintNs = MXATTN_ROLE_WAIT_HINT_NS;

template <int D, int T, bool NV = false>
struct Cfg {
    static constexpr int kStages = 4;
    static constexpr int kTiles = 2;                  // query tiles per CTA
    static constexpr int kRows = 128 * kTiles;        // query rows per CTA
    static constexpr int kSoftThreads = 128 * kTiles;
    static constexpr int kProducerWarp = 4 * kTiles;
    static constexpr int kMmaWarp = 4 * kTiles + 1;  // S issuer (and TMEM allocator)
    static constexpr int kPvWarp = 4 * kTiles + 2;   // PV issuer
    // A third, full warpgroup holds the producer and the two MMA-issuing warps
    // (plus one idle warp) so registers can move between warpgroups with setmaxnreg.
    static constexpr int kThreads = kSoftThreads + 128;
    // Launch: kThreads x kLaunchRegs registers (ptxas's cap for 12 warps, 3 per
    // sub-partition).  Split: softmax warpgroups kSoftRegs, the other kRoleRegs;
    // 2 x 128 x 224 + 128 x 56 == 384 x 168.
    static constexpr uint32_t kLaunchRegs = 168;
    static constexpr uint32_t kSoftRegs = 224;
    static constexpr uint32_t kRoleRegs = 56;
    static_assert(kTiles * 128 * kSoftRegs + 128 * kRoleRegs == kThreads * kLaunchRegs, "register split");
    static constexpr int kQBytes = 128 * D / 2;
    static constexpr int kKBytes = T * D / 2;
    static constexpr int kVRows = D + 16;  // V^T rows + a row of ones + 15 zero rows
    static constexpr int kVLoadBytes = D * T / 2;
    static constexpr int kVStride = ((kVRows * T / 2) + 1023) / 1024 * 1024;
    static constexpr int kPBytes = 128 * T / 2;
    // Scale factors travel in 512-byte atoms (128 rows x 4 scale bytes, the
    // order tcgen05 reads them).  MXFP4 (block 32): one atom covers a 128-row
    // tile for any d or kv_tile here.  NVFP4 (block 16): one atom per 64
    // columns of the contraction axis.
    static constexpr int kQAtoms = NV ? D / 64 : 1;                       // Q and K, per 128-row group
    static constexpr int kVAtoms = NV ? T / 64 : 1;                       // V^T per key tile; P per tile
    static constexpr int kQsfBytes = 512 * kQAtoms;
    static constexpr int kVsfGroupBytes = NV ? 1024 : 512;               // V^T scales per 128 tokens in HBM
    static constexpr int kVsfBytes = 512 * kVAtoms;                      // V^T scales loaded per key tile
    static constexpr int kPsfBytes = 512 * kVAtoms;
    static constexpr int kSfBytes = 512;                                  // one atom
    // TMEM slots for the K and V^T scale factors (NVFP4's larger scales leave room for two)
    static constexpr int kSfSlots = NV ? 2 : kStages;
    static constexpr int kOCols = D + 16;
    // Of the 16 exponential pairs of a 32-column block, this many go to the FMA
    // pipe instead of the MUFU: with PNQ (the code-only stand-in for 2^w,
    // exp2_code_sat_x2) 7 for MXFP4 and 8 for NVFP4, whose block scales add MUFU
    // work of their own; 6 without PNQ (the full polynomial, exp2_fma_x2).  Pair q
    // is one of them when (q * n) mod 16 < n, which spreads them evenly.
    __host__ __device__ static constexpr bool fma_pair(int q, bool pnq) {
        const int n = pnq ? (NV ? 8 : 7) : 6;  // measured best for each format
        return (q * n) % 16 < n;
    }

    static constexpr uint32_t kQKLayout = (D == 128) ? kLayoutSw64 : kLayoutSw32;
    static constexpr uint32_t kQKSbo = 8 * D / 2;
    static constexpr uint32_t kPVLayout = (T == 128) ? kLayoutSw64 : kLayoutSw32;
    static constexpr uint32_t kPVSbo = 8 * T / 2;

    // shared memory (offsets from a 1024-aligned base)
    static constexpr int kOffQ = 0;                                     // [kTiles]
    static constexpr int kOffK = kOffQ + kTiles * kQBytes;              // [kStages]
    static constexpr int kOffV = kOffK + kStages * kKBytes;             // [kStages]
    static constexpr int kOffP = kOffV + kStages * kVStride;            // [kTiles]
    static constexpr int kOffQsf = kOffP + kTiles * kPBytes;            // [kTiles]
    static constexpr int kOffKsf = kOffQsf + kTiles * kQsfBytes;        // [kStages]
    static constexpr int kOffVsf = kOffKsf + kStages * kQsfBytes;       // [kStages]
    static constexpr int kOffPsf = kOffVsf + kStages * kVsfBytes;       // [kTiles]
    static constexpr int kOffVsfConst = kOffPsf + kTiles * kPsfBytes;
    static constexpr int kOffBar = kOffVsfConst + kSfBytes;
    // barriers: q, k_full[S], k_empty[S], v_full[S], v_empty[S],
    //           s_full[kTiles], s_loaded[kTiles], p_full[kTiles], o_done[kTiles], drain
    static constexpr int kNumBars = 1 + 4 * kStages + 4 * kTiles + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemUsed = kOffMisc + 16;
    // >= 116 KB keeps one CTA per SM, so the 512-column TMEM allocation never waits
    static constexpr int kSmemBytes = (kSmemUsed + 1024 > 116 * 1024) ? kSmemUsed + 1024 : 116 * 1024;

    // TMEM columns: one S buffer shared by both tiles, then O per tile, then scale factors
    static constexpr uint32_t kColS = 0;
    static constexpr uint32_t kColO = T;  // + t * kOCols
    // (4 columns per atom; a V^T atom also has 4 columns for rows 128..255)
    static constexpr uint32_t kColQsf = (T + kTiles * kOCols + 3) / 4 * 4;  // + 4 kQAtoms t
    static constexpr uint32_t kColKsf = kColQsf + 4 * kQAtoms * kTiles;     // + 4 kQAtoms slot
    static constexpr uint32_t kColPsf = kColKsf + 4 * kQAtoms * kSfSlots;   // + 4 kVAtoms t
    static constexpr uint32_t kColVsf = kColPsf + 4 * kVAtoms * kTiles;     // + 8 kVAtoms slot
    static constexpr uint32_t kColsUsed = kColVsf + 8 * kVAtoms * kSfSlots;
    static_assert(kColsUsed <= 512, "TMEM budget");
    static_assert(kSmemUsed + 1024 <= 227 * 1024, "shared memory budget");
};

struct KParams {
    const uint8_t* q_sf;
    const uint8_t* k_sf;
    const uint8_t* v_sf;
    float* O;
    uint32_t* status;
    int N;
    int nq2;     // CTAs (pairs of query tiles) per head
    int nkv;     // key tiles per head
    int groups;  // 128-row scale groups per head
    float kq;    // softmax_scale * log2(e)
    // log2 Qmax of P's scale boundary when Qmax < 8 (the kernel's OCP form ignores it):
    // block exponent e = ceil(x - log2 Qmax) with x the log2 of the block's largest exponential.
    float log2q;
    // NVFP4: the second-level scales g of Q, K, V per (batch, head), [3][BH]
    const float* gs;
    int BH;
};

// Maximum of 32 values as a depth-4 tree of 3-input max instructions.
__device__ __forceinline__ float block_max32(const float* v) {
    float t[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) t[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    t[10] = fmaxf(v[30], v[31]);
    const float u0 = fmax3(t[0], t[1], t[2]);
    const float u1 = fmax3(t[3], t[4], t[5]);
    const float u2 = fmax3(t[6], t[7], t[8]);
    const float u3 = fmaxf(t[9], t[10]);
    return fmax3(u0, u1, fmaxf(u2, u3));
}

// Maximum of 16 values.
__device__ __forceinline__ float block_max16(const float* v) {
    const float t0 = fmax3(v[0], v[1], v[2]), t1 = fmax3(v[3], v[4], v[5]), t2 = fmax3(v[6], v[7], v[8]);
    const float t3 = fmax3(v[9], v[10], v[11]), t4 = fmax3(v[12], v[13], v[14]);
    return fmax3(fmax3(t0, t1, t2), t3, fmaxf(t4, v[15]));
}

__device__ __forceinline__ uint64_t sf_desc(const void* p) {
    // 32 rows x 16 bytes, rows contiguous: core matrices of 8 rows 128 bytes apart
    return smem_desc(smem_u32(p), 0, 128, kLayoutNone);
}

template <int D, int T, bool PNQ, bool NV, bool OCP>
__global__ void __launch_bounds__(Cfg<D, T, NV>::kThreads, 1)
    mxattn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ KParams p) {
    using C = Cfg<D, T, NV>;
    constexpr int S = C::kStages;
    constexpr int NT = C::kTiles;
    extern __shared__ uint8_t smem_raw[];
    // Aligned by an offset from the shared array itself, so every derived pointer
    // keeps the shared address space (32-bit addressing, nothing held as a generic pointer).
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sP = smem + C::kOffP;
    uint8_t* sQsf = smem + C::kOffQsf;
    uint8_t* sKsf = smem + C::kOffKsf;
    uint8_t* sVsf = smem + C::kOffVsf;
    uint8_t* sPsf = smem + C::kOffPsf;
    uint8_t* sVsfConst = smem + C::kOffVsfConst;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* bar_q = bars;
    uint64_t* bar_k_full = bars + 1;
    uint64_t* bar_k_empty = bar_k_full + S;
    uint64_t* bar_v_full = bar_k_empty + S;
    uint64_t* bar_v_empty = bar_v_full + S;
    uint64_t* bar_s_full = bar_v_empty + S;      // [NT]
    uint64_t* bar_s_loaded = bar_s_full + NT;    // [NT]
    uint64_t* bar_p_full = bar_s_loaded + NT;    // [NT]
    uint64_t* bar_o_done = bar_p_full + NT;      // [NT]
    uint64_t* bar_drain = bar_o_done + NT;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int bh = blockIdx.x / p.nq2;
    const int qp = blockIdx.x % p.nq2;  // pair index: rows [256 qp, 256 qp + 256)
    const int nkv = p.nkv;

    if (tid == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(bar_k_full + s, 1);
            mbar_init(bar_k_empty + s, 1);
            mbar_init(bar_v_full + s, 1);
            mbar_init(bar_v_empty + s, 1);
        }
        for (int t = 0; t < NT; ++t) {
            mbar_init(bar_s_full + t, 1);
            mbar_init(bar_s_loaded + t, 128);
            mbar_init(bar_p_full + t, 128);
            mbar_init(bar_o_done + t, 1);
        }
        mbar_init(bar_drain, 2);  // one commit from each MMA-issuing thread
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    // Constant rows of every V^T stage: row D = ones (E2M1 1.0 = code 2), rows D+1.. = 0.
    for (int idx = tid; idx < S * 16 * (T / 2) / 4; idx += C::kThreads) {
        const int s = idx / (16 * (T / 2) / 4);
        const int w = idx % (16 * (T / 2) / 4);
        const int row = D + w / (T / 8);
        reinterpret_cast<uint32_t*>(sV + s * C::kVStride + D * (T / 2))[w] = (row == D) ? 0x22222222u : 0u;
    }
    // Scale factors of V^T rows 128..255 (only used when D = 128): all 1 (E8M0 2^0, or E4M3 1.0).
    for (int idx = tid; idx < 128; idx += C::kThreads)
        reinterpret_cast<uint32_t*>(sVsfConst)[idx] = NV ? 0x38383838u : 0x7F7F7F7Fu;
    fence_proxy_async_smem();
    if (warp == C::kMmaWarp) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = *tmem_holder;

    // Each warpgroup's code lives entirely in its own branch (register budget
    // set by setmaxnreg at the top of the branch), ending with a block-wide
    // named barrier after which the MMA warp frees TMEM.
    if (warp >= 4 * NT) {
        warpgroup_regs_dec<C::kRoleRegs>();
        // The producer and the MMA issuer run their loops with the whole warp,
        // so the loop state stays warp-uniform; one elected lane (fixed for
        // the kernel) issues every copy and tcgen05 instruction.
        const bool leader = elect_one_sync();
        auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag, p.status, kTimeoutCode,
                                                             kTimeoutNs, kRoleWaitHintNs));
        };
        if (warp == C::kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
            int k_issued = 0, v_issued = 0;
            if (leader) {
                mbar_arrive_expect_tx(bar_q, NT * (C::kQBytes + C::kQsfBytes));
                for (int t = 0; t < NT; ++t) {
                    const int g = 2 * qp + t;  // 128-row group of tile t (may lie past N: zero-filled)
                    tma_load_3d(sQ + t * C::kQBytes, &tmQ, bar_q, 0, g * 128, bh);
                    const int gs = g < p.groups ? g : p.groups - 1;  // keep the scale copy inside the buffer
                    bulk_load(sQsf + t * C::kQsfBytes, p.q_sf + (static_cast<size_t>(bh) * p.groups + gs) * C::kQsfBytes,
                              C::kQsfBytes, bar_q);
                }
            }
            __syncwarp();
            for (int j = 0; j < nkv; ++j) {
                const int s = j % S;
                const uint32_t n = j / S;
                const size_t grp = static_cast<size_t>(bh) * p.groups + (j * T) / 128;
                if (j >= S && !wait(bar_k_empty + s, (n - 1) & 1)) break;
                if (leader) {
                    mbar_arrive_expect_tx(bar_k_full + s, C::kKBytes + C::kQsfBytes);
                    tma_load_3d(sK + s * C::kKBytes, &tmK, bar_k_full + s, 0, j * T, bh);
                    bulk_load(sKsf + s * C::kQsfBytes, p.k_sf + grp * C::kQsfBytes, C::kQsfBytes, bar_k_full + s);
                }
                __syncwarp();
                k_issued = j + 1;
                if (j >= S && !wait(bar_v_empty + s, (n - 1) & 1)) break;
                if (leader) {
                    mbar_arrive_expect_tx(bar_v_full + s, C::kVLoadBytes + C::kVsfBytes);
                    tma_load_3d(sV + s * C::kVStride, &tmV, bar_v_full + s, j * (T / 2), 0, bh);
                    // NVFP4 with 64-key tiles: the key tile is one of the group's two 64-token atoms
                    const size_t vsf_off = grp * C::kVsfGroupBytes + ((NV && T == 64) ? (j & 1) * 512 : 0);
                    bulk_load(sVsf + s * C::kVsfBytes, p.v_sf + vsf_off, C::kVsfBytes, bar_v_full + s);
                }
                __syncwarp();
                v_issued = j + 1;
            }
            // Drain: every copy the leader issued must land before the CTA exits.
            // On the normal path these phases completed long ago and the waits return at once.
            int dummy = 0;
            volatile int* no_abort = &dummy;
            mbar_wait_bounded(bar_q, 0, no_abort, p.status, kTimeoutCode, kTimeoutNs);
            // only the newest tile of each stage can still be in flight
            for (int j = k_issued - S < 0 ? 0 : k_issued - S; j < k_issued; ++j)
                mbar_wait_bounded(bar_k_full + j % S, (j / S) & 1, no_abort, p.status, kTimeoutCode, kTimeoutNs);
            for (int j = v_issued - S < 0 ? 0 : v_issued - S; j < v_issued; ++j)
                mbar_wait_bounded(bar_v_full + j % S, (j / S) & 1, no_abort, p.status, kTimeoutCode, kTimeoutNs);
            __syncwarp();
    } else if (warp == C::kMmaWarp || warp == C::kPvWarp) {
        // ------------------------------------------------------------ MMA issuers (S: warp 9, PV: warp 10)
            const uint32_t t_s = tbase + C::kColS;
            // Shared-memory descriptors of the first buffer of each operand; a buffer
            // b bytes further on is the descriptor plus b >> 4 (start-address field).
            const uint64_t qdesc0 = smem_desc(smem_u32(sQ), 16, C::kQKSbo, C::kQKLayout);
            const uint64_t kdesc0 = smem_desc(smem_u32(sK), 16, C::kQKSbo, C::kQKLayout);
            const uint64_t pdesc0 = smem_desc(smem_u32(sP), 16, C::kPVSbo, C::kPVLayout);
            const uint64_t vdesc0 = smem_desc(smem_u32(sV), 16, C::kPVSbo, C::kPVLayout);
            const uint64_t ksf0 = sf_desc(sKsf), vsf0 = sf_desc(sVsf), psf0 = sf_desc(sPsf);
            // S_t(j) = Q_t K(j)^T into the shared S buffer.  Tile A's issue also
            // waits for K(j) and copies its scales; tile B reuses both.
            auto issue_s = [&](int t, int j) -> bool {
                const int s = j % S;
                const uint32_t n = j / S;
                const int slot = j % C::kSfSlots;
                if (t == 0 && !wait(bar_k_full + s, n & 1)) return false;
                tc_fence_after_sync();  // after the K wait, or after the wait for the S buffer to be read
                const uint64_t qdesc = qdesc0 + static_cast<uint32_t>(t * (C::kQBytes >> 4));
                const uint64_t kdesc = kdesc0 + static_cast<uint32_t>(s * (C::kKBytes >> 4));
                const uint32_t ksf_col = tbase + C::kColKsf + 4 * C::kQAtoms * slot;
                const uint32_t ksf = ksf_col + ((T == 64) ? 2 * (j & 1) : 0);  // rows 64..127 of the group: +2 columns
                if (leader) {
                    if (t == 0) {
#pragma unroll
                        for (int a = 0; a < C::kQAtoms; ++a)
                            tc_cp_sf(ksf_col + 4 * a, ksf0 + static_cast<uint32_t>((s * C::kQsfBytes + 512 * a) >> 4));
                    }
#pragma unroll
                    for (int kk = 0; kk < D / 64; ++kk) {
                        if constexpr (NV)
                            tc_mma_nvf4(t_s, qdesc + 2 * kk, kdesc + 2 * kk, nvf4_idesc(T),
                                        tbase + C::kColQsf + 4 * C::kQAtoms * t + 4 * kk, ksf + 4 * kk, kk > 0 ? 1u : 0u);
                        else
                            tc_mma_mxf4(t_s, qdesc + 2 * kk, kdesc + 2 * kk, mxf4_idesc(T, 2 * kk, 2 * kk),
                                        tbase + C::kColQsf + 4 * t, ksf, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(bar_s_full + t);
                    if (t == NT - 1) tc_commit(bar_k_empty + s);
                }
                __syncwarp();
                return true;
            };
            // O_t += P_t V(j).  Tile A's issue waits for V(j) and copies its scales.
            auto issue_pv = [&](int t, int j) -> bool {
                const int s = j % S;
                const uint32_t n = j / S;
                const int slot = j % C::kSfSlots;
                if (!wait(bar_p_full + t, j & 1)) return false;
                if (t == 0 && !wait(bar_v_full + s, n & 1)) return false;
                tc_fence_after_sync();
                const uint64_t pdesc = pdesc0 + static_cast<uint32_t>(t * (C::kPBytes >> 4));
                const uint64_t vdesc = vdesc0 + static_cast<uint32_t>(s * (C::kVStride >> 4));
                const uint32_t psf_col = tbase + C::kColPsf + 4 * C::kVAtoms * t;
                const uint32_t vsf_col = tbase + C::kColVsf + 8 * C::kVAtoms * slot;
                if (leader) {
#pragma unroll
                    for (int a = 0; a < C::kVAtoms; ++a)
                        tc_cp_sf(psf_col + 4 * a, psf0 + static_cast<uint32_t>((t * C::kPsfBytes + 512 * a) >> 4));
                    if (t == 0) {
#pragma unroll
                        for (int a = 0; a < C::kVAtoms; ++a)
                            tc_cp_sf(vsf_col + 8 * a, vsf0 + static_cast<uint32_t>((s * C::kVsfBytes + 512 * a) >> 4));
                    }
#pragma unroll
                    for (int kk = 0; kk < T / 64; ++kk) {
                        if constexpr (NV) {
                            tc_mma_nvf4(tbase + C::kColO + t * C::kOCols, pdesc + 2 * kk, vdesc + 2 * kk,
                                        nvf4_idesc(D + 16), psf_col + 4 * kk, vsf_col + 8 * kk,
                                        (j > 0 || kk > 0) ? 1u : 0u);
                        } else {
                            const uint32_t sfb_id = (T == 64) ? 2u * (j & 1) : 2u * kk;
                            tc_mma_mxf4(tbase + C::kColO + t * C::kOCols, pdesc + 2 * kk, vdesc + 2 * kk,
                                        mxf4_idesc(D + 16, 2 * kk, sfb_id), psf_col, vsf_col,
                                        (j > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(bar_o_done + t);
                    if (t == NT - 1) tc_commit(bar_v_empty + s);
                }
                __syncwarp();
                return true;
            };
            if (warp == C::kMmaWarp) {
                // S issuer.  Order: S_A(0); S_B(0) once A has read the S buffer; then per
                // key tile j: S_A(j) once B has read S_B(j-1), S_B(j) once A has read S_A(j).
                bool ok = wait(bar_q, 0);
                if (ok) {
                    tc_fence_after_sync();
                    if (leader) {
                        for (int t = 0; t < NT; ++t)
                            for (int a = 0; a < C::kQAtoms; ++a)
                                tc_cp_sf(tbase + C::kColQsf + 4 * C::kQAtoms * t + 4 * a,
                                         sf_desc(sQsf + t * C::kQsfBytes + 512 * a));
                    }
                    __syncwarp();
                }
                ok = ok && issue_s(0, 0);
                ok = ok && wait(bar_s_loaded + 0, 0) && issue_s(1, 0);
                for (int j = 1; ok && j < nkv; ++j) {
                    ok = wait(bar_s_loaded + 1, (j - 1) & 1) && issue_s(0, j);
                    ok = ok && wait(bar_s_loaded + 0, j & 1) && issue_s(1, j);
                }
            } else {
                // PV issuer: the constant V^T scales of rows 128..255 once (d = 128), then
                // O_A += P_A V(j) and O_B += P_B V(j) for every key tile, as each P arrives.
                if (D == 128) {
                    if (leader)
                        for (int slot = 0; slot < C::kSfSlots; ++slot)
                            for (int a = 0; a < C::kVAtoms; ++a)
                                tc_cp_sf(tbase + C::kColVsf + 8 * C::kVAtoms * slot + 8 * a + 4, sf_desc(sVsfConst));
                    __syncwarp();
                }
                for (int j = 0; j < nkv; ++j) {
                    if (!issue_pv(0, j)) break;
                    if (!issue_pv(1, j)) break;
                }
            }
            // Drain: wait for every MMA / copy both issuers made before TMEM is freed
            // (bar_drain completes once each issuing thread's commit has arrived).
            if (leader) tc_commit(bar_drain);
            __syncwarp();
            int dummy = 0;
            mbar_wait_bounded(bar_drain, 0, &dummy, p.status, kTimeoutCode, kTimeoutNs);
            __syncwarp();
    }
    tc_fence_before_sync();
    named_barrier_sync(1, C::kThreads);
    if (warp == C::kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tbase, 512);
    }
    } else {
        warpgroup_regs_inc<C::kSoftRegs>();
        // ------------------------------------------------------------ softmax (thread = query row of tile t)
        const int t = warp >> 2;
        const int row = tid & 127;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_o = tbase + lane_base + C::kColO + t * C::kOCols;
        // NVFP4: S and O come out of the tensor core in units of the second-level
        // scales 6 g (Q, K, V) and 6 * 448 (P); fold them into kq and the epilogue.
        float kq = p.kq;
        float o_unit = 1.f;
        if constexpr (NV) {
            const float Gq = __fmul_rn(6.f, p.gs[bh]), Gk = __fmul_rn(6.f, p.gs[p.BH + bh]);
            kq = p.kq / (Gq * Gk);
            o_unit = __fmul_rn(6.f, p.gs[2 * p.BH + bh]);
        }
        const float kq8 = 0.125f * kq;  // exact: the stand-in's map of w onto [0, 1] scales by 1/8
        const float log2q = p.log2q;
        const int valid_last = p.N - (nkv - 1) * T;
        uint8_t* sPt = sP + t * C::kPBytes;
        uint8_t* sPsft = sPsf + t * C::kPsfBytes;
        float m_run = -INFINITY;
        float l_run = 0.f;  // PNQ off: the row sum of the unquantized exponentials
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_s_full + t, j & 1, abort_flag, p.status,
                                                            kTimeoutCode, kTimeoutNs))) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            uint32_t sr[T / 64][64];
#pragma unroll
            for (int c = 0; c < T / 64; ++c) tmem_ld64_sync(tbase + lane_base + C::kColS + 64 * c, sr[c]);
            float sv[T];
#pragma unroll
            for (int c = 0; c < T / 64; ++c)
#pragma unroll
                for (int i = 0; i < 64; ++i) sv[64 * c + i] = __uint_as_float(sr[c][i]);
            tc_fence_before_sync();
            mbar_arrive(bar_s_loaded + t);
            if (j == nkv - 1 && valid_last < T) {
#pragma unroll
                for (int i = 0; i < T; ++i)
                    if (i >= valid_last) sv[i] = -INFINITY;
            }
            constexpr int NBM = NV ? T / 16 : T / 32;  // blocks of P (16 or 32 keys)
            float bm[NBM];
#pragma unroll
            for (int k = 0; k < NBM; ++k) bm[k] = NV ? block_max16(sv + 16 * k) : block_max32(sv + 32 * k);
            float tmax = bm[0];
#pragma unroll
            for (int k = 1; k < NBM; ++k) tmax = fmaxf(tmax, bm[k]);
            const float m_new = fmaxf(m_run, tmax);
            const bool rescale = (j > 0) && (m_new > m_run);
            const float alpha = rescale ? ex2_approx((m_run - m_new) * kq) : 1.f;

            uint32_t pw[T / 8];
            uint32_t sfw[C::kVAtoms];
#pragma unroll
            for (int a = 0; a < C::kVAtoms; ++a) sfw[a] = 0u;
            float lsum = 0.f;
            // Per block of P: `nbias[k]` turns s * kq into the log2 of the element as it
            // enters the E2M1 rounding, `back[k]` brings a rounded value back to exp(s - m_new).
            // `nb8[k]` = (nbias[k] + 2) / 8 is the same bias for the code-only stand-in
            // (exp2_code_sat_x2), formed with one rounding like nbias.
            float nbias[NBM], nb8[NBM], back[NBM];
            if constexpr (NV) {
                // NVFP4 P (blocks of 16 keys): scale sb = E4M3(pmax * 448) with pmax the block's
                // largest exponential, element = exp(s - m_new) * 2688 / sb.  A block whose scale
                // rounds to 0 holds values below 2.3e-6 and is left unscaled (all its codes are 0).
#pragma unroll
                for (int k = 0; k < NBM; ++k) {
                    const uint32_t sb = nv_p_block_scale((bm[k] - m_new) * kq);
                    const float sbv = e4m3_decode(sb);
                    // log2(2688 / sbv) split as an exact integer plus a fraction rounded once:
                    // ei = 138 - (biased fp32 exponent of sbv), fr = log2(1.3125) - log2(significand).
                    float ei, fr;
                    nv_p_scale_log2_parts(sbv, ei, fr);
                    nbias[k] = fmaf(-m_new, kq, sb ? fr + ei : 0.f);
                    if constexpr (PNQ) nb8[k] = fmaf(-m_new, kq8, sb ? fmaf(fr, 0.125f, fmaf(ei, 0.125f, 0.25f)) : 0.25f);
                    if constexpr (!PNQ) back[k] = sb ? sbv * (1.f / 2688.f) : 1.f;
                    sfw[k / 4] |= sb << (8 * (k % 4));
                }
            } else {
                // MXFP4 P: the block's largest exponential is 2^x with x = (bm - m_new) * kq; the
                // scale rule is applied to it in the log domain (no exponential needed), and each
                // element is then 2^(s*kq - (m*kq + e)), already divided by the block scale 2^e.
                // bm - m_new is exactly 0 for the block holding the row max, so the OCP boundary
                // at integer x is decided exactly there.
#pragma unroll
                for (int k = 0; k < NBM; ++k) {
                    uint32_t byte;
                    const float ef = p_block_exp<OCP>(bm[k] - m_new, kq, log2q, byte);
                    nbias[k] = fmaf(-m_new, kq, -ef);                                      // -(m kq + e), one rounding
                    if constexpr (PNQ) nb8[k] = fmaf(-m_new, kq8, fmaf(ef, -0.125f, 0.25f));  // (nbias + 2) / 8, one rounding
                    if constexpr (!PNQ) back[k] = byte ? __uint_as_float(byte << 23) : __uint_as_float(0x00400000u);
                    sfw[0] |= byte << (8 * k);
                }
            }
            // Elements, 8 at a time (group gg: keys 8 gg .. 8 gg + 7, P block gg / (NV ? 2 : 4)).
#pragma unroll
            for (int gg = 0; gg < T / 8; ++gg) {
                const int k = NV ? gg / 2 : gg / 4;
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    float w0, w1;
                    if (!C::fma_pair(4 * (gg % 4) + i / 2, PNQ)) {  // MUFU
                        ffma2_bcast(w0, w1, sv[8 * gg + i], sv[8 * gg + i + 1], kq, nbias[k]);
                        f[i] = ex2_approx(w0);
                        f[i + 1] = ex2_approx(w1);
                    } else if constexpr (PNQ) {  // FMA pipe: only the E2M1 code is kept
                        exp2_code_sat_x2(sv[8 * gg + i], sv[8 * gg + i + 1], kq8, nb8[k], f[i], f[i + 1]);
                    } else {                     // FMA pipe: the value enters the row sum
                        ffma2_bcast(w0, w1, sv[8 * gg + i], sv[8 * gg + i + 1], kq, nbias[k]);
                        exp2_fma_x2(w0, w1, f[i], f[i + 1]);
                    }
                }
                if constexpr (!PNQ) {
                    float gsum = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) gsum += f[i];
                    lsum = fmaf(gsum, back[k], lsum);
                }
                pw[gg] = pack_e2m1x8(f);
            }
            // The P buffer and O are free once the previous P*V of this tile finished.
            if (j > 0) {
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_o_done + t, (j - 1) & 1, abort_flag, p.status,
                                                                kTimeoutCode, kTimeoutNs))) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
            }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t r[64];
                    tmem_ld64_sync(t_o + 64 * c, r);
#pragma unroll
                    for (int i = 0; i < 64; i += 2) fmul2_bcast(r[i], r[i + 1], r[i], r[i + 1], alpha);
                    tmem_st64(t_o + 64 * c, r);
                }
                if constexpr (PNQ)
                    tmem_st1(t_o + D, __float_as_uint(__uint_as_float(tmem_ld1_sync(t_o + D)) * alpha));
                tmem_st_wait();
            }
            // P row -> shared memory in the swizzled K-major layout the MMA reads.
            {
                uint8_t* prow = sPt + row * (T / 2);
#pragma unroll
                for (int c = 0; c < T / 32; ++c) {
                    const int phys = (T == 128) ? (c ^ ((row >> 1) & 3)) : (c ^ ((row >> 2) & 1));
                    *reinterpret_cast<uint4*>(prow + 16 * phys) =
                        make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
                }
#pragma unroll
                for (int a = 0; a < C::kVAtoms; ++a)
                    reinterpret_cast<uint32_t*>(sPsft + 512 * a)[(row & 31) * 4 + (row >> 5)] = sfw[a];
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(bar_p_full + t);
            if constexpr (!PNQ) l_run = fmaf(l_run, alpha, lsum);
            m_run = m_new;
        }
        // Epilogue: O / l for the valid rows.
        if (ok && __all_sync(0xffffffffu, mbar_wait_bounded(bar_o_done + t, (nkv - 1) & 1, abort_flag, p.status,
                                                             kTimeoutCode, kTimeoutNs))) {
            tc_fence_after_sync();
            // NVFP4: O and the PNQ row sum carry P's factor 2688 and O also V's 6 g.
            const float l = PNQ ? __uint_as_float(tmem_ld1_sync(t_o + D)) : (NV ? 2688.f * l_run : l_run);
            const float inv_l = 1.f / (l * o_unit);
            const int qrow = qp * C::kRows + t * 128 + row;
            float* out = p.O + (static_cast<size_t>(bh) * p.N + qrow) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32_sync(t_o + 32 * c, r);
                if (qrow < p.N) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(out + 32 * c + i) =
                            make_float4(__uint_as_float(r[i]) * inv_l, __uint_as_float(r[i + 1]) * inv_l,
                                        __uint_as_float(r[i + 2]) * inv_l, __uint_as_float(r[i + 3]) * inv_l);
                }
            }
        }
        tc_fence_before_sync();
        named_barrier_sync(1, C::kThreads);
    }
}

// 3-D byte tensor [outer, rows, inner_bytes] with a (box_inner x box_rows x 1) box.
bool encode_map(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows, uint64_t outer,
                uint32_t box_inner, uint32_t box_rows) {
    auto fn = tensor_map_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {inner_bytes, rows, outer};
    cuuint64_t strides[2] = {inner_bytes, inner_bytes * rows};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = (box_inner == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, int T, bool PNQ, bool NV, bool OCP>
cudaError_t launch_impl(const AttnArgs& a, cudaStream_t stream) {
    using C = Cfg<D, T, NV>;
    static bool attr_set = false;
    if (!attr_set) {
        // The setmaxnreg split assumes the launch allocates exactly kLaunchRegs per
        // thread; with fewer, the softmax warpgroups' increase could never be met.
        cudaFuncAttributes fa{};
        cudaError_t e = cudaFuncGetAttributes(&fa, mxattn_fwd_kernel<D, T, PNQ, NV, OCP>);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != static_cast<int>(C::kLaunchRegs)) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(mxattn_fwd_kernel<D, T, PNQ, NV, OCP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int npad = (a.N + 31) / 32 * 32;
    CUtensorMap tq, tk, tv;
    if (!encode_map(&tq, a.q_codes, D / 2, a.N, a.BH, D / 2, 128) ||
        !encode_map(&tk, a.k_codes, D / 2, a.N, a.BH, D / 2, T) ||
        !encode_map(&tv, a.vt_codes, npad / 2, D, a.BH, T / 2, D))
        return cudaErrorInvalidValue;
    KParams kp{};
    kp.q_sf = a.q_sf;
    kp.k_sf = a.k_sf;
    kp.v_sf = a.v_sf;
    kp.O = a.O;
    kp.status = a.status;
    kp.N = a.N;
    kp.nq2 = (a.N + C::kRows - 1) / C::kRows;
    kp.nkv = (a.N + T - 1) / T;
    kp.groups = (a.N + 127) / 128;
    kp.kq = static_cast<float>(static_cast<double>(a.softmax_scale) * 1.4426950408889634);
    kp.log2q = OCP ? 0.f : static_cast<float>(std::log2(static_cast<double>(a.qmax)));
    kp.gs = a.gs;
    kp.BH = static_cast<int>(a.BH);
    dim3 grid(static_cast<unsigned>(a.BH * kp.nq2));
    mxattn_fwd_kernel<D, T, PNQ, NV, OCP><<<grid, C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, kp);
    return cudaGetLastError();
}

}  // namespace

template <int D, int T>
cudaError_t launch_pnq(const AttnArgs& a, cudaStream_t stream) {
    if (a.nv)
        return a.pnq ? launch_impl<D, T, true, true, false>(a, stream) : launch_impl<D, T, false, true, false>(a, stream);
    if (a.qmax >= 8.f)  // the OCP rule
        return a.pnq ? launch_impl<D, T, true, false, true>(a, stream) : launch_impl<D, T, false, false, true>(a, stream);
    return a.pnq ? launch_impl<D, T, true, false, false>(a, stream) : launch_impl<D, T, false, false, false>(a, stream);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t stream) {
    if (a.d == 128 && a.kv_tile == 128) return launch_pnq<128, 128>(a, stream);
    if (a.d == 128 && a.kv_tile == 64) return launch_pnq<128, 64>(a, stream);
    if (a.d == 64 && a.kv_tile == 128) return launch_pnq<64, 128>(a, stream);
    if (a.d == 64 && a.kv_tile == 64) return launch_pnq<64, 64>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace mxattn
