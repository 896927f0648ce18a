"""Pins for the oracle's rotary embedding + FP8 append (CPU only).

Checked against: torch's own float32 -> bfloat16 conversion, exact special
angles (0 and 90 degrees), an independent complex-number evaluation in
float64, float64 evaluation with one rounding per operation (the stated
float32 arithmetic), the rotation-group properties (composition, relative
position of the dot product), and the plain append of the rotated K."""

import numpy as np
import torch

from oracle import e4m3, paged, rope


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(10.0),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.0078125, 3.0e38, -3.0e38, 1e-40, 65504.0],
                 np.float32),
        # exact halfway cases between two bf16 values (ties to even)
        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(rope.bf16_round(x).view(np.uint32), want.view(np.uint32))


def test_special_angles_are_exact():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 128)).astype(np.float32)
    one, zero = np.ones(64, np.float32), np.zeros(64, np.float32)
    assert np.array_equal(rope.rotate(x, one, zero), x)                # angle 0
    r = rope.rotate(x, zero, one)                                       # 90 degrees
    assert np.array_equal(r[:, :64], -x[:, 64:]) and np.array_equal(r[:, 64:], x[:, :64])


def test_matches_complex_multiplication():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 3, 64)).astype(np.float32)
    ang = rng.uniform(-10, 10, (7, 1, 32))
    c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    got = rope.rotate(x, c, s).astype(np.float64)
    z = (x[..., :32].astype(np.float64) + 1j * x[..., 32:].astype(np.float64)) * \
        (c.astype(np.float64) + 1j * s.astype(np.float64))
    want = np.concatenate([z.real, z.imag], axis=-1)
    assert np.max(np.abs(got - want)) <= 1e-6 * np.max(np.abs(want))


def test_one_rounding_per_operation():
    """The float32 result equals float64 evaluation with a rounding to float32
    after each product and after the sum (no fused multiply-add)."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2000, 64)).astype(np.float32) * np.float32(3)
    ang = rng.uniform(0, 6.3, (2000, 32))
    c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    f32 = lambda a: np.asarray(a, np.float64).astype(np.float32).astype(np.float64)  # noqa: E731
    x1, x2 = x[:, :32].astype(np.float64), x[:, 32:].astype(np.float64)
    c64, s64 = c.astype(np.float64), s.astype(np.float64)
    o1 = f32(f32(x1 * c64) - f32(x2 * s64))
    o2 = f32(f32(x2 * c64) + f32(x1 * s64))
    got = rope.rotate(x, c, s)
    assert np.array_equal(got, np.concatenate([o1, o2], axis=-1).astype(np.float32))
    # and it differs from a fused evaluation somewhere (the reading matters)
    fused = (x1 * c64 - f32(x2 * s64)).astype(np.float32)
    assert np.any(fused != got[:, :32])


def test_rotation_properties():
    rng = np.random.default_rng(5)
    D = 128
    theta = 10000.0 ** (-np.arange(D // 2) * 2.0 / D)
    q, k = rng.standard_normal((2, D))

    def rot64(x, pos):
        a = pos * theta
        return rope.rotate(x, np.cos(a), np.sin(a)).astype(np.float64)

    # relative position: <R(m) q, R(n) k> depends on m - n only (float32 rounding)
    d1 = rot64(q, 17) @ rot64(k, 5)
    d2 = rot64(q, 1017) @ rot64(k, 1005)
    assert abs(d1 - d2) <= 1e-4 * np.linalg.norm(q) * np.linalg.norm(k)
    # the norm of each (i, i + D/2) pair is kept
    r = rot64(q, 333)
    assert np.allclose(r[:64] ** 2 + r[64:] ** 2, q[:64] ** 2 + q[64:] ** 2, rtol=1e-5)


def test_rope_append_rotates_k_only_and_rounds_q():
    rng = np.random.default_rng(6)
    B, n_new, Hq, Hkv, D, ps, P = 2, 3, 4, 2, 128, 16, 6
    qkv = torch.from_numpy(rng.standard_normal((B, n_new, Hq + 2 * Hkv, D)).astype(np.float32))
    qkv = qkv.to(torch.bfloat16).float().numpy()
    table = np.zeros((64, D), np.float32)
    a = rng.uniform(0, 6.3, (64, D // 2))
    table[:, :D // 2], table[:, D // 2:] = np.cos(a), np.sin(a)
    ks, vs = np.array([0.02, 0.03], np.float32), np.array([0.01, 0.04], np.float32)
    bt = np.array([[0, 1, 2], [3, 4, 5]], np.int32)
    start = np.array([14, 30], np.int32)
    kp0 = np.zeros((P, Hkv, ps, D), np.uint8)
    vp0 = np.zeros((P, Hkv, ps, D), np.uint8)
    q_out, kp, vp = rope.rope_append(kp0, vp0, qkv, Hq, Hkv, table, ks, vs, bt, start, ps)
    for b in range(B):
        for t in range(n_new):
            pos = start[b] + t
            c, s = table[pos, :64], table[pos, 64:]
            page, slot = paged.slot_of(bt, b, pos, ps)
            for h in range(Hkv):
                kr = rope.rotate(qkv[b, t, Hq + h], c, s)
                assert np.array_equal(kp[page, h, slot], e4m3.encode(kr, ks[h]))
                assert np.array_equal(vp[page, h, slot], e4m3.encode(qkv[b, t, Hq + Hkv + h], vs[h]))
            for h in range(Hq):
                want = torch.from_numpy(rope.rotate(qkv[b, t, h], c, s)).to(torch.bfloat16).float()
                assert np.array_equal(q_out[b, t, h], want.numpy())
