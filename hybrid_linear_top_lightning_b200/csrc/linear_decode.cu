// lisa_linear_decode on sm_100a: one recurrent step of the linear-attention
// branch (LISA, arXiv 2607.19358v1, Sec. 3.1 "Linear Attention", Sec. 3.3
// Eq. 3-4): S <- S + phi(k)^T v, o = phi(q) S (divided by phi(q).z_new in the
// elu+1 mode, z_new = z + phi(k)), for bf16 activations with head dim 128 and
// an fp32 state.
//
// k_linear_decode: one CTA (128 threads) per (sequence, KV head, 32 value
// columns): the state slice S[:, c0:c0+32] (16 KB) comes into shared memory by
// 16-byte cp.async copies, then the decode step's own slice routine
// (decode_linear.cuh) advances it, writes it back and reads out the group's
// query heads.  Every slice of a head reads the old z, so the elu+1 mode
// advances z in a second small kernel.  HBM-bound: the state is read and
// written once (2 x 64 KB per KV head).
#include "linear_decode.cuh"

#include "decode_linear.cuh"
#include "lisa_internal.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;
constexpr int kMaxGroup = 8;  // query heads per KV head this path takes
constexpr int kSlices = dec::kLaD / dec::kLaCols;

struct LinDecParams {
    const bf16* q_L;  // [B][H_q][128]
    const bf16* k_L;  // [B][H_kv][128]
    const bf16* v_L;  // [B][H_kv][128]
    float* S;         // [B][H_kv][128][128] in/out
    float* z;         // [B][H_kv][128] (elu+1 mode) read here, advanced by k_z_advance
    bf16* olin;       // [B][H_q][128]
    int H_q, H_kv, group, phi;
};

__global__ void __launch_bounds__(dec::kLaThreads) k_linear_decode(const LinDecParams P) {
    __shared__ __align__(16) float s_slice[dec::kLaD * dec::kLaCols];
    __shared__ float fk[dec::kLaD], fq[kMaxGroup * dec::kLaD], vcol[dec::kLaCols], zloc[dec::kLaD],
        den[kMaxGroup];
    const int c0 = (int)(blockIdx.x % kSlices) * dec::kLaCols;
    const int bg = (int)(blockIdx.x / kSlices);
    const int b = bg / P.H_kv, g = bg % P.H_kv;
    const float* Sg = P.S + (int64_t)bg * dec::kLaD * dec::kLaD;
    constexpr int kQuads = dec::kLaCols / 4;  // 16-byte pieces per state row of the slice
    for (int e = threadIdx.x; e < dec::kLaD * kQuads; e += dec::kLaThreads) {
        const int i = e / kQuads, c4 = e % kQuads;
        ptx::cp_async_16(s_slice + i * dec::kLaCols + 4 * c4, Sg + (int64_t)i * dec::kLaD + c0 + 4 * c4);
    }
    ptx::cp_async_commit();
    dec::linear_slice(P, 0, b, g, c0, s_slice, fk, fq, vcol, zloc, den);
}

// z <- z + phi(k), once every slice has read the old z (elu+1 mode)
__global__ void __launch_bounds__(256) k_z_advance(const LinDecParams P, int total) {
    const int i = blockIdx.x * 256 + threadIdx.x;
    if (i < total) P.z[i] += dec::feat(P.phi, __bfloat162float(P.k_L[i]));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fast_linear_decode_supported(const Shape& s, const void* q, const void* k, const void* v,
                                  const float* S) {
    return s.dtype == LISA_BF16 && s.d == dec::kLaD && s.T == 1 && s.group <= kMaxGroup &&
           aligned16(q) && aligned16(k) && aligned16(v) && aligned16(S);
}

cudaError_t fast_linear_decode(const Shape& s, const void* q, const void* k, const void* v, float* S,
                               float* z, void* o_lin, cudaStream_t st) {
    LinDecParams P;
    P.q_L = static_cast<const bf16*>(q);
    P.k_L = static_cast<const bf16*>(k);
    P.v_L = static_cast<const bf16*>(v);
    P.S = S;
    P.z = z;
    P.olin = static_cast<bf16*>(o_lin);
    P.H_q = s.H_q;
    P.H_kv = s.H_kv;
    P.group = s.group;
    P.phi = s.phi;
    const int64_t ctas = (int64_t)s.B * s.H_kv * kSlices;
    if (ctas == 0) return cudaSuccess;
    if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
    k_linear_decode<<<(unsigned)ctas, dec::kLaThreads, 0, st>>>(P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || s.phi != LISA_PHI_ELU1_NORM) return e;
    const int total = s.B * s.H_kv * dec::kLaD;
    k_z_advance<<<(total + 255) / 256, 256, 0, st>>>(P, total);
    return cudaGetLastError();
}

}  // namespace lisa
