// Step 4 (prefill) -- gate-weighted combine back to token order, and the unit-RMS chaining
// helper for stacked layers.  Both are pure HBM streams: 16-byte vectors, one pass.
//
//   combine: y[t, :] = sum_{j<k} g[t,j] * o_sorted[inv_pos[t*k+j], :] (+ o_sorted[inv_pos[T*k+t], :])
//            fp32 accumulation in j order (shared term last), one RNE rounding to bf16.
//            Gather form (each token pulls its k rows), so no atomics and a fixed order.
//   unit_rms: out[t, :] = bf16(y[t, :] / sqrt(mean(y[t, :]^2) + eps)), fp32.
#include "kernels.h"

namespace ftmoe {

// DEP: launched as a programmatic dependent of the expert kernel that writes o (decode
// batches): the routing (inv_pos, gates; final before that kernel started) is read before
// the wait, o after it, and the next kernel may be scheduled at once.
template <bool DEP>
__global__ void __launch_bounds__(256) combine_kernel(int T, int H, int k, int S, int R, const uint16_t* __restrict__ o,
                                                      const int32_t* __restrict__ inv_pos, const float* __restrict__ gw,
                                                      uint16_t* __restrict__ y) {
    if (DEP) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int t = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;     // 16-byte column vector index
    const int P = T * k;
    int pos[kMaxTopK + 1];
    float wgt[kMaxTopK + 1];
    int nterm = 0;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) { pos[nterm] = inv_pos[t * k + j]; wgt[nterm] = gw[t * k + j]; ++nterm; }
    }
    if (S) { pos[nterm] = inv_pos[P + t]; wgt[nterm] = 1.0f; ++nterm; }
    if (DEP) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (c * 8 >= H) return;
    uint4 v[kMaxTopK + 1];
#pragma unroll
    for (int j = 0; j < kMaxTopK + 1; ++j) {
        if (j < nterm) {
            int p = pos[j];
            v[j] = (p >= 0 && p < R) ? ldg_nc_v4(o + size_t(p) * H + c * 8) : make_uint4(0, 0, 0, 0);
        }
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK + 1; ++j) {
        if (j < nterm) {
            const float g = wgt[j];
            acc[0] = fmaf(g, bf16lo(v[j].x), acc[0]); acc[1] = fmaf(g, bf16hi(v[j].x), acc[1]);
            acc[2] = fmaf(g, bf16lo(v[j].y), acc[2]); acc[3] = fmaf(g, bf16hi(v[j].y), acc[3]);
            acc[4] = fmaf(g, bf16lo(v[j].z), acc[4]); acc[5] = fmaf(g, bf16hi(v[j].z), acc[5]);
            acc[6] = fmaf(g, bf16lo(v[j].w), acc[6]); acc[7] = fmaf(g, bf16hi(v[j].w), acc[7]);
        }
    }
    uint4 out = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
    *reinterpret_cast<uint4*>(y + size_t(t) * H + c * 8) = out;
}

cudaError_t launch_combine(int T, int H, int k, int S, int R, const uint16_t* o, const int32_t* inv_pos,
                           const float* gw, uint16_t* y, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    dim3 grid((H / 8 + 255) / 256, T);
    combine_kernel<false><<<grid, 256, 0, st>>>(T, H, k, S, R, o, inv_pos, gw, y);
    return cudaGetLastError();
}

cudaError_t launch_combine_dependent(int T, int H, int k, int S, int R, const uint16_t* o, const int32_t* inv_pos,
                                     const float* gw, uint16_t* y, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((H / 8 + 255) / 256, T);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel<true>, T, H, k, S, R, o, inv_pos, gw, y);
}

__global__ void __launch_bounds__(256) unit_rms_kernel(int H, const uint16_t* in, uint16_t* out, float eps) {
    __shared__ float red[8];
    const int t = blockIdx.x, tid = threadIdx.x;
    const uint4* row = reinterpret_cast<const uint4*>(in + size_t(t) * H);
    const int nv = H / 8;
    float ss = 0.f;
    for (int c = tid; c < nv; c += 256) {
        uint4 u = row[c];
        float f[8] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y), bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w)};
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float inv = 1.0f / sqrtf(tot / float(H) + eps);
    __syncthreads();   // every read of `in` is done before an aliasing `out` is written
    uint4* orow = reinterpret_cast<uint4*>(out + size_t(t) * H);
    for (int c = tid; c < nv; c += 256) {
        uint4 u = row[c];
        orow[c] = make_uint4(pack_bf16x2(bf16lo(u.x) * inv, bf16hi(u.x) * inv), pack_bf16x2(bf16lo(u.y) * inv, bf16hi(u.y) * inv),
                             pack_bf16x2(bf16lo(u.z) * inv, bf16hi(u.z) * inv), pack_bf16x2(bf16lo(u.w) * inv, bf16hi(u.w) * inv));
    }
}

cudaError_t launch_unit_rms(int T, int H, const uint16_t* in, uint16_t* out, float eps, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    unit_rms_kernel<<<T, 256, 0, st>>>(H, in, out, eps);
    return cudaGetLastError();
}

}  // namespace ftmoe
