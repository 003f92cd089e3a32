// vtranspose.cu -- V [B*Hkv][T][D] -> V^T [B*Hkv][D][T8] (bf16), T8 = T rounded up to 8, the
// padding zero-filled.  Stage 2 feeds V^T to the tensor cores as the K-major B operand of
// O += P V (keys contiguous per head dim), which the MMA reads at full rate; V itself would be
// an MN-major operand, measured at about 60% of that rate for these shapes.  TMA fetches 64
// keys of all 128 dims of a chunk as one 128-byte-swizzled box.  HBM-bound: 2 * B*Hkv*T*D*2
// bytes per call.
#include "dash_common.cuh"
#include "kernels.cuh"

namespace dash {

constexpr int kTrTile = 64;

template <int D>
__global__ void __launch_bounds__(256) k_vtranspose(const __nv_bfloat16 *__restrict__ v,
                                                    __nv_bfloat16 *__restrict__ vt, int T, int T8,
                                                    int t_base) {
    __shared__ __nv_bfloat16 tile[kTrTile][kTrTile + 2];
    const int bg = blockIdx.z, t0 = t_base + blockIdx.x * kTrTile, d0 = blockIdx.y * kTrTile;
    const __nv_bfloat16 *src = v + (long long)bg * T * D;
    __nv_bfloat16 *dst = vt + (long long)bg * D * T8;
    for (int i = threadIdx.x; i < kTrTile * kTrTile; i += 256) {
        const int r = i / kTrTile, c = i % kTrTile;          // r: key, c: dim
        const int t = t0 + r;
        tile[r][c] = t < T ? src[(long long)t * D + d0 + c] : __float2bfloat16(0.f);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kTrTile * kTrTile; i += 256) {
        const int r = i / kTrTile, c = i % kTrTile;          // r: dim, c: key
        const int t = t0 + c;
        if (t < T8) dst[(long long)(d0 + r) * T8 + t] = tile[c][r];
    }
}

cudaError_t launch_vtranspose(const void *v, void *vt, int BHkv, int T, int D, cudaStream_t st,
                              int k_begin, int k_end) {
    const int T8 = (T + 7) & ~7;
    if (k_end <= 0 || k_end >= T) k_end = T8;            // the range reaching T covers the padding
    if (k_begin < 0 || (k_begin % kTrTile) != 0 || k_begin >= k_end) return cudaErrorInvalidValue;
    dim3 grid((k_end - k_begin + kTrTile - 1) / kTrTile, D / kTrTile, BHkv);
    if (D == 128)
        k_vtranspose<128><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(v),
                                                reinterpret_cast<__nv_bfloat16 *>(vt), T, T8, k_begin);
    else if (D == 64)
        k_vtranspose<64><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(v),
                                               reinterpret_cast<__nv_bfloat16 *>(vt), T, T8, k_begin);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace dash
