// Quaternion arithmetic for the IsoQuant block rotation (arXiv 2603.28430,
// abstract): the 4 coordinates 4m .. 4m+3 of a vector form the quaternion
// v = v0 + v1 i + v2 j + v3 k, which turns into qL v conj(qR) (IsoQuant-Full;
// qR = 1 gives IsoQuant-Fast).  Rotation parameters are stored per block as
// 8 floats, qL then qR, each (w, x, y, z).
#pragma once

namespace axr {

struct Quat {
    float w, x, y, z;
};

// Hamilton product a b (i^2 = j^2 = k^2 = ijk = -1)
__device__ __forceinline__ Quat qmul(const Quat &a, const Quat &b)
{
    return {a.w * b.w - a.x * b.x - a.y * b.y - a.z * b.z, a.w * b.x + a.x * b.w + a.y * b.z - a.z * b.y,
            a.w * b.y - a.x * b.z + a.y * b.w + a.z * b.x, a.w * b.z + a.x * b.y - a.y * b.x + a.z * b.w};
}

// qL and conj(qR) of block m (quats 16-byte aligned)
__device__ __forceinline__ void block_quats(const float *quats, int m, Quat &qL, Quat &qRc)
{
    const float4 l = __ldg(reinterpret_cast<const float4 *>(quats) + 2 * m);
    const float4 r = __ldg(reinterpret_cast<const float4 *>(quats) + 2 * m + 1);
    qL = {l.x, l.y, l.z, l.w};
    qRc = {r.x, -r.y, -r.z, -r.w};
}

// qL = conj(qR) = 1: what a debug build substitutes for a block it may not read
__device__ __forceinline__ void unit_quats(Quat &qL, Quat &qRc)
{
    qL = {1.0f, 0.0f, 0.0f, 0.0f};
    qRc = {1.0f, 0.0f, 0.0f, 0.0f};
}

__device__ __forceinline__ Quat block_rotate(const Quat &qL, const Quat &qRc, const Quat &v)
{
    return qmul(qmul(qL, v), qRc);
}

}  // namespace axr
