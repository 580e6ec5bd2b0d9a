"""The seeded input generator (moe_inputs), checked on the host.

Both the CUDA path's tests and the oracle draw their inputs from it, so a
mistake there would hide from every parity test.  These pin what its recipe
states: the E4M3 block quantisation (scale = block amax / 448, codes rounded
to nearest, all-zero block at scale 1), the router-logit bias for skewed
loads, the per-tensor seeding and the synthetic routing helpers."""
import math

import numpy as np
import torch

import moe_inputs

E4M3_MIN_NORMAL = 2.0 ** -6   # E4M3: 4 exponent bits (bias 7), 3 mantissa bits
E4M3_HALF_SUBNORMAL_STEP = 2.0 ** -10


def _block_matrix():
    """[256, 384] bf16: 2 x 3 blocks of 128 x 128 at very different magnitudes,
    one all-zero, one whose small entries land among E4M3's subnormals."""
    g = torch.Generator().manual_seed(7)
    w = torch.randn((256, 384), generator=g)
    mags = [[1.0, 3e-3, 50.0], [0.0, 1.0, 1e-8]]
    for i in range(2):
        for j in range(3):
            w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128] *= mags[i][j]
    # block (1, 1): one large entry, the rest 1e-5 of it -> codes below 2^-6
    blk = w[128:256, 128:256]
    blk.mul_(1e-5)
    blk[5, 9] = 2.0
    return w.to(torch.bfloat16)


def test_e4m3_block_scales_are_the_block_amax_over_448():
    w = _block_matrix()
    q, s = moe_inputs.quantize_e4m3_blocks(w)
    assert q.dtype == torch.float8_e4m3fn and q.shape == w.shape
    assert s.dtype == torch.float32 and s.shape == (2, 3)
    wf = w.float()
    for i in range(2):
        for j in range(3):
            b = wf[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            amax = float(b.abs().max())
            if amax == 0.0:
                assert float(s[i, j]) == 1.0
                assert not q[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128].float().any()
            else:
                assert float(s[i, j]) == float(torch.tensor(amax, dtype=torch.float32) / 448.0)
                # the largest entry of the block takes the largest finite code
                qb = q[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128].float()
                r, c = divmod(int(b.abs().argmax()), 128)
                assert abs(float(qb[r, c])) == 448.0
                assert float(qb.abs().max()) == 448.0


def test_e4m3_codes_round_to_nearest_within_half_a_step():
    """|q s - w| <= s * half a code step at |w / s|: 2^-4 |w / s| among normal
    codes (3 mantissa bits), 2^-10 among subnormal ones."""
    w = _block_matrix()
    q, s = moe_inputs.quantize_e4m3_blocks(w)
    sf = s.repeat_interleave(128, 0).repeat_interleave(128, 1).double()
    v = w.double() / sf
    err = (q.double() * sf - w.double()).abs()
    bound = torch.maximum(v.abs() * 2.0 ** -4, torch.full_like(v, E4M3_HALF_SUBNORMAL_STEP)) * sf
    assert bool((err <= bound * (1 + 1e-6)).all())
    # the bound is tight enough to catch truncation: some entries must round up
    trunc = torch.sign(v) * torch.floor(v.abs() * 8) / 8
    assert bool(((q.double() - trunc).abs() > 0).any())
    # and the subnormal range was reached
    sub = (v.abs() < E4M3_MIN_NORMAL) & (v != 0)
    assert int(sub.sum()) > 1000


def test_e4m3_codes_are_round_half_even_on_exact_ties():
    """Values exactly halfway between two codes go to the even mantissa."""
    # block amax 448 -> scale exactly 1, so w is the pre-rounding value
    w = torch.zeros((128, 128), dtype=torch.float32)
    w[0, 0] = 448.0
    # between 1.0 (mantissa 000) and 1.125 (001): 1.0625 -> 1.0 (even)
    # between 1.125 (001) and 1.25 (010): 1.1875 -> 1.25 (even)
    # between subnormals 2^-9 (001) and 2^-8 (010): 1.5 * 2^-9 -> 2^-8 (even)
    w[1, :3] = torch.tensor([1.0625, 1.1875, 1.5 * 2.0 ** -9])
    q, s = moe_inputs.quantize_e4m3_blocks(w.to(torch.bfloat16))
    assert float(s[0, 0]) == 1.0
    assert q[1, :3].float().tolist() == [1.0, 1.25, 2.0 ** -8]


def test_zipf_bias_closed_form():
    """b_e = 2 ln(1 / rank_e^1.1), rank_e = e + 1: at equal logits the router's
    probabilities fall off as rank^-2.2, expert 0 the hottest."""
    E = 512
    b = moe_inputs.zipf_bias(E, "cpu").double()
    assert b.dtype == torch.float64 and b.shape == (E,)
    assert float(b[0]) == 0.0
    for e in (1, 2, 9, 255, 511):
        assert abs(float(b[e]) - 2.0 * math.log(1.0 / (e + 1) ** 1.1)) < 1e-5
    p = torch.softmax(b, 0)
    assert abs(float(p[1] / p[0]) - 2.0 ** -2.2) < 1e-5
    assert bool((b[1:] < b[:-1]).all())


def test_each_tensor_has_its_own_seeded_stream():
    a = moe_inputs.make_inputs(40, 64, 6, 2, 32, 32, act="bf16", w="bf16", seed=3)
    b = moe_inputs.make_inputs(40, 64, 6, 2, 32, 32, act="bf16", w="bf16", seed=3)
    names = ("x", "w_r", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd")
    for n in names:
        assert torch.equal(getattr(a, n), getattr(b, n)), n
    # a new batch (x_seed) re-draws x alone
    c = moe_inputs.make_inputs(40, 64, 6, 2, 32, 32, act="bf16", w="bf16", seed=3, x_seed=4)
    assert not torch.equal(a.x, c.x)
    for n in names[1:]:
        assert torch.equal(getattr(a, n), getattr(c, n)), n
    # a tensor's draw does not depend on the shapes of the ones before it
    d = moe_inputs.make_inputs(40, 64, 9, 2, 32, 32, act="bf16", w="bf16", seed=3)
    assert torch.equal(a.x, d.x)
    assert torch.equal(a.s_wg, d.s_wg)
    # the streams differ from tensor to tensor
    assert not torch.equal(a.wg, a.wu)
    # N(0, 1) activations, N(0, 0.02^2) weights
    big = moe_inputs.make_inputs(512, 256, 8, 2, 128, 128, act="f32", w="f32", seed=1)
    assert abs(float(big.x.std()) - 1.0) < 0.01
    for n in ("w_r", "wg", "wd", "s_wu"):
        assert abs(float(getattr(big, n).std()) - 0.02) < 0.001, n
    assert big.x.dtype == torch.float32 and a.x.dtype == torch.bfloat16


def test_fp8_inputs_carry_a_packed_scale_per_block():
    inp = moe_inputs.make_inputs(16, 256, 3, 2, 128, 256, act="bf16", w="fp8", seed=2)
    assert inp.wg.dtype == torch.float8_e4m3fn and inp.s_wd.dtype == torch.float8_e4m3fn
    n_routed = 3 * (1 * 2) * 3          # gate, up, down: 2 blocks each per expert
    n_shared = 2 * 2 + 2 * 2 + 2 * 2    # I_s = 256, d = 256: 4 blocks each
    assert inp.scales.shape == (n_routed + n_shared,)
    # every block's largest code is +-448, so max |q| * s is that block's amax
    for m in (inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd):
        mf = m.float().reshape(*m.shape[:-2], m.shape[-2] // 128, 128, m.shape[-1] // 128, 128)
        assert bool((mf.abs().amax(dim=(-3, -1)) == 448.0).all())


def test_random_routing_draws_distinct_experts_and_positive_weights():
    T, E, k = 300, 11, 4
    ids, w = moe_inputs.random_routing(T, E, k, seed=9)
    assert ids.dtype == torch.int32 and ids.shape == (T, k)
    a = ids.numpy()
    assert a.min() >= 0 and a.max() < E
    assert all(len(set(r)) == k for r in a.tolist())
    assert w.dtype == torch.float32 and bool((w > 0).all())
    # every expert gets picked at this size
    assert set(np.unique(a).tolist()) == set(range(E))


def test_random_groups_offsets_are_the_running_sum():
    sizes = [3, 0, 129, 1, 0, 40]        # 5 routed groups + the shared one
    offs = moe_inputs.random_groups(5, sizes)
    assert offs.dtype == torch.int32
    assert offs.tolist() == [0, 3, 3, 132, 133, 133, 173]
