// host.cu -- mxattn_forward_host: MXFP4 attention from host buffers to host
// buffers, with the copies pipelined against the attention.
//
// The (batch, head) slices are independent problems, so the call processes
// them in groups: the copy to the device of group i+1 and the copy back of
// group i-1 overlap the attention of group i.  Copies run on two streams of
// their own (one per direction, since a PCIe link carries both directions at
// once), the attention on the caller's stream; events order the three.  The
// streams and events are created for the call and released by the runtime
// once the GPU has finished with them, so the library keeps no state between
// calls.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "kernels.cuh"
#include "mxattn.h"

#define MXATTN_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kDefaultGroups = 16;

// Default schedule for BH slices in n groups: the first and the last group one
// slice each (the copy in of the first group and the copy out of the last are
// the only transfers nothing overlaps), the others as equal as possible.
std::vector<int> default_groups(int64_t BH, int n) {
    std::vector<int> g;
    if (n <= 0) n = kDefaultGroups;
    if (n > BH) n = static_cast<int>(BH);
    if (n < 3 || BH < 3) {
        const int64_t per = (BH + n - 1) / n;
        for (int64_t c = 0; c < BH; c += per) g.push_back(static_cast<int>(BH - c < per ? BH - c : per));
        return g;
    }
    const int64_t mid = BH - 2;
    const int k = n - 2;
    g.push_back(1);
    for (int i = 0; i < k; ++i) g.push_back(static_cast<int>(mid / k + (i < mid % k ? 1 : 0)));
    g.push_back(1);
    return g;
}

bool make_groups(int64_t BH, const int* sizes, int ngroups, std::vector<int>* out) {
    if (sizes == nullptr) {
        if (ngroups < 0) return false;
        *out = default_groups(BH, ngroups);
        return true;
    }
    if (ngroups < 1) return false;
    int64_t sum = 0;
    for (int i = 0; i < ngroups; ++i) {
        if (sizes[i] < 1) return false;
        sum += sizes[i];
    }
    if (sum != BH) return false;
    out->assign(sizes, sizes + ngroups);
    return true;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

MXATTN_API size_t mxattn_forward_host_workspace_size(int B, int H, int N, int d, const int* group_sizes,
                                                     int ngroups) {
    if (B < 1 || H < 1) return 0;
    std::vector<int> g;
    if (!make_groups(static_cast<int64_t>(B) * H, group_sizes, ngroups, &g)) return 0;
    int gmax = 0;
    for (int s : g) gmax = s > gmax ? s : gmax;
    return mxattn_workspace_size(1, gmax, N, d);
}

MXATTN_API mxattn_status mxattn_forward_host(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                             int kv_tile, int pnq, mxattn_rule rule, float softmax_scale, float* O,
                                             void* q_dev, void* k_dev, void* v_dev, float* o_dev, void* workspace,
                                             size_t workspace_bytes, const int* group_sizes, int ngroups,
                                             mxattn_stream_t stream) {
    if (rule != MXATTN_RULE_OCP && rule != MXATTN_RULE_UOS) return MXATTN_ERR_INVALID;
    mxattn_status st = mxattn::check_attention_shape(B, H, N, d, kv_tile, pnq, O);
    if (st != MXATTN_OK) return st;
    if (Q == nullptr || K == nullptr || V == nullptr || q_dev == nullptr || k_dev == nullptr || v_dev == nullptr ||
        o_dev == nullptr || workspace == nullptr)
        return MXATTN_ERR_INVALID;
    if (!aligned(q_dev, 16) || !aligned(k_dev, 16) || !aligned(v_dev, 16) || !aligned(o_dev, 16) ||
        !aligned(workspace, 256))
        return MXATTN_ERR_INVALID;
    const int64_t BH = static_cast<int64_t>(B) * H;
    std::vector<int> groups;
    if (!make_groups(BH, group_sizes, ngroups, &groups)) return MXATTN_ERR_INVALID;
    if (workspace_bytes < mxattn_forward_host_workspace_size(B, H, N, d, group_sizes, ngroups))
        return MXATTN_ERR_INVALID;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t in_slice = static_cast<size_t>(N) * d * 2;   // bytes of one (b, h) slice of Q, K or V
    const size_t out_slice = static_cast<size_t>(N) * d * 4;  // of O
    cudaStream_t h2d = nullptr, d2h = nullptr;
    std::vector<cudaEvent_t> evs;
    auto event = [&](cudaEvent_t* e) -> bool {
        if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
        evs.push_back(*e);
        return true;
    };
    bool ok = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t start = nullptr;
    // The staging buffers may still be in use by earlier work on `stream`.
    ok = ok && event(&start) && cudaEventRecord(start, s) == cudaSuccess &&
         cudaStreamWaitEvent(h2d, start, 0) == cudaSuccess && cudaStreamWaitEvent(d2h, start, 0) == cudaSuccess;
    int64_t c0 = 0;
    for (size_t gi = 0; ok && gi < groups.size(); ++gi) {
        const int n = groups[gi];
        const size_t in_off = static_cast<size_t>(c0) * in_slice, out_off = static_cast<size_t>(c0) * out_slice;
        auto dev_in = [&](void* p) { return static_cast<uint8_t*>(p) + in_off; };
        auto host_in = [&](const void* p) { return static_cast<const uint8_t*>(p) + in_off; };
        cudaEvent_t loaded = nullptr, done = nullptr;
        ok = cudaMemcpyAsync(dev_in(q_dev), host_in(Q), n * in_slice, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
             cudaMemcpyAsync(dev_in(k_dev), host_in(K), n * in_slice, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
             cudaMemcpyAsync(dev_in(v_dev), host_in(V), n * in_slice, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
             event(&loaded) && cudaEventRecord(loaded, h2d) == cudaSuccess &&
             cudaStreamWaitEvent(s, loaded, 0) == cudaSuccess;
        if (!ok) break;
        st = mxattn_forward(dev_in(q_dev), dev_in(k_dev), dev_in(v_dev), 1, n, N, d, kv_tile, pnq, rule,
                            softmax_scale, reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(o_dev) + out_off),
                            workspace, workspace_bytes, stream);
        if (st != MXATTN_OK) break;
        ok = event(&done) && cudaEventRecord(done, s) == cudaSuccess && cudaStreamWaitEvent(d2h, done, 0) == cudaSuccess &&
             cudaMemcpyAsync(reinterpret_cast<uint8_t*>(O) + out_off, reinterpret_cast<uint8_t*>(o_dev) + out_off,
                             n * out_slice, cudaMemcpyDeviceToHost, d2h) == cudaSuccess;
        c0 += n;
    }
    // Whatever was enqueued, `stream` waits for both copy streams before it goes on.
    cudaEvent_t in_end = nullptr, out_end = nullptr;
    bool joined = h2d != nullptr && d2h != nullptr && event(&in_end) && cudaEventRecord(in_end, h2d) == cudaSuccess &&
                  cudaStreamWaitEvent(s, in_end, 0) == cudaSuccess && event(&out_end) &&
                  cudaEventRecord(out_end, d2h) == cudaSuccess && cudaStreamWaitEvent(s, out_end, 0) == cudaSuccess;
    // Released by the runtime once the work recorded on them has completed.
    for (cudaEvent_t e : evs) cudaEventDestroy(e);
    if (h2d != nullptr) cudaStreamDestroy(h2d);
    if (d2h != nullptr) cudaStreamDestroy(d2h);
    if (st != MXATTN_OK) return st;
    return (ok && joined) ? MXATTN_OK : MXATTN_ERR_CUDA;
}
