"""GPU parity of fp4_quantize / fp4_dequantize against the CPU oracle.

Packed nibbles, scale bytes (tile layout, padding included) and the NVFP4
tensor scale must be bit-exact; dequantized fp32 values too (both sides do the
same IEEE fp32 operations), and bf16 output is the RNE rounding of them.
"""
import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

from helpers import bf16_tensor_bits, to_dev_bf16, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp4():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_microscaling_quantization_b200 import build
    build.build()
    import fp4_microscaling_quantization_b200 as m
    return m


def check_quantize(fp4, orc, x, fmt, hk=0, tie=0, rule=0, gscale=None, x_dev=None, search=0):
    import torch
    rows, cols = x.shape
    xd = to_dev_bf16(x) if x_dev is None else x_dev
    gs = None if gscale is None else torch.tensor([gscale], dtype=torch.float32, device="cuda")
    q, s, g = fp4.quantize(xd, fmt, hadamard_k=hk, round=tie, mx_scale_rule=rule, gscale=gs, scale_search=search)
    torch.cuda.synchronize()
    oq, os_, og = orc.quantize(x, fmt, hadamard_k=hk, tie=tie, mx_rule=rule, gscale=gscale, search=search)
    q_np, s_np = to_np(q), to_np(s)
    bad = np.argwhere(q_np != oq)
    assert bad.size == 0, f"nibbles differ at {bad[:4].tolist()}: gpu {q_np[tuple(bad[0])]:#x} oracle {oq[tuple(bad[0])]:#x}"
    os_atoms = orc.scales_to_atoms(os_)
    assert s_np.shape == os_atoms.shape
    sbad = np.flatnonzero(s_np != os_atoms)
    assert sbad.size == 0, f"scales differ at {sbad[:4].tolist()}"
    if fmt == fp4.FP4_NVFP4:
        assert np.float32(to_np(g)[0]) == np.float32(og), (to_np(g)[0], og)
    return q, s, g, (oq, os_, og)


SHAPES = [(1, 32), (3, 96), (130, 512), (257, 1024), (64, 4096), (37, 3104), (5, 32736)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_parity_shapes(fp4, orc, shape, fmt):
    rows, cols = shape
    rng = np.random.default_rng(rows * 7 + cols)
    v = rng.laplace(0, 1, shape).astype(np.float32)
    v[rng.random(shape) < 0.01] *= 20
    check_quantize(fp4, orc, inputs.f32_to_bf16_bits(v), fmt)


@pytest.mark.parametrize("hk", [16, 32, 64, 128])
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_parity_rotated(fp4, orc, hk, fmt):
    x = inputs.rotate_acts(rows=136, cols=1024, seed=hk)
    check_quantize(fp4, orc, x, fmt, hk=hk)


@pytest.mark.parametrize("fmt,tie,rule", [(0, 1, 0), (0, 0, 1), (0, 1, 1), (1, 1, 0)])
def test_quantize_parity_modes(fp4, orc, fmt, tie, rule):
    x = inputs.quant_sweep(rows=40, cols=2048, seed=9)
    check_quantize(fp4, orc, x, fmt, hk=32, tie=tie, rule=rule)
    check_quantize(fp4, orc, x, fmt, hk=0, tie=tie, rule=rule)


def edge_tensor():
    """Rows of special values: zeros, -0, bf16 subnormals, exact E2M1 ties
    under a power-of-two scale, saturation, lone outliers, huge values."""
    rows = []
    rows.append(np.zeros(64, np.float32))
    rows.append(-np.zeros(64, np.float32))
    sub = np.array([(i + 1) * 2.0 ** -133 for i in range(64)], np.float32)  # bf16 subnormals
    rows.append(sub * np.where(np.arange(64) % 2, -1, 1))
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 8, np.float32)
    rows.append(ties * np.where(np.arange(64) % 3 == 0, -1, 1))   # block max 6 -> scale 1
    rows.append(ties * 2.0 ** 20)
    r = np.full(64, 1e-3, np.float32)
    r[5] = 1e4
    r[40] = -3e5
    rows.append(r)
    rows.append(np.linspace(-3e38, 3e38, 64).astype(np.float32))
    rows.append(np.full(64, -1.0, np.float32))
    x = np.stack(rows)
    return inputs.f32_to_bf16_bits(x)


@pytest.mark.parametrize("fmt,tie", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_quantize_edge_cases(fp4, orc, fmt, tie):
    x = edge_tensor()
    check_quantize(fp4, orc, x, fmt, tie=tie)
    check_quantize(fp4, orc, x[:6], fmt, tie=tie, hk=64)


@pytest.mark.parametrize("gscale", [1.0, 1e-3, 1e-30, 7.5e2, 3e30])
def test_nvfp4_given_global_scale(fp4, orc, gscale):
    """Offline s_g: saturation (tiny s_g), underflow to zero scales (huge s_g)."""
    x = inputs.quant_sweep(rows=16, cols=512, seed=3)
    check_quantize(fp4, orc, x, 1, gscale=gscale)


def test_all_zero_tensor_nvfp4(fp4, orc):
    x = np.zeros((5, 64), np.uint16)
    q, s, g, _ = check_quantize(fp4, orc, x, 1)
    assert to_np(g)[0] == 1.0


def test_strided_input(fp4, orc):
    import torch
    x = inputs.quant_sweep(rows=33, cols=512, seed=4)
    big = np.zeros((33, 640), np.uint16)
    big[:, :512] = x
    xd = to_dev_bf16(big)[:, :512]
    assert xd.stride(0) == 640
    for fmt in (0, 1):
        check_quantize(fp4, orc, x, fmt, x_dev=xd)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("hk", [0, 32, 128])
@pytest.mark.parametrize("bf16", [0, 1])
def test_dequantize_parity(fp4, orc, fmt, hk, bf16):
    import torch
    x = inputs.rotate_acts(rows=130, cols=512, seed=5)
    q, s, g, (oq, os_, og) = check_quantize(fp4, orc, x, fmt, hk=hk)
    out = fp4.dequantize(q, s, g, fmt, hadamard_k=hk, out_dtype=bf16)
    torch.cuda.synchronize()
    ref = orc.dequantize(oq, os_, og, fmt, hadamard_k=hk)
    if bf16:
        got = bf16_tensor_bits(out)
        want = inputs.f32_to_bf16_bits(ref)
        assert np.array_equal(got, want)
    else:
        got = to_np(out)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # leaving the values rotated: dequantize without the inverse rotation
    if hk:
        out2 = fp4.dequantize(q, s, g, fmt, hadamard_k=0)
        ref2 = orc.dequantize(oq, os_, og, fmt, hadamard_k=0)
        assert np.array_equal(to_np(out2).view(np.uint32), ref2.view(np.uint32))


@pytest.mark.parametrize("fmt", [0, 1])
def test_full_size_quant_sweep(fp4, orc, fmt):
    """1024 x 131072 heavy-tailed tensor: whole-tensor parity at the
    benchmark's size and launch configuration."""
    import torch
    x = inputs.quant_sweep()
    check_quantize(fp4, orc, x, fmt)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("hk", [0, 16, 128])
def test_full_size_rotate(fp4, orc, fmt, hk):
    """8192 x 4096 activations with outlier channels, rotated then quantized."""
    x = inputs.rotate_acts()
    check_quantize(fp4, orc, x, fmt, hk=hk)


def test_reuses_output_buffers(fp4, orc):
    import torch
    x = inputs.quant_sweep(rows=8, cols=256, seed=1)
    xd = to_dev_bf16(x)
    q, s, g = fp4.quantize(xd, 1)
    q2, s2, g2 = fp4.quantize(xd, 1, out=(torch.empty_like(q), torch.empty_like(s), torch.empty_like(g)))
    assert torch.equal(q, q2) and torch.equal(s, s2) and torch.equal(g, g2)


@pytest.mark.parametrize("row", range(8))
@pytest.mark.parametrize("fmt", [0, 1])
def test_edge_rows_alone(fp4, orc, row, fmt):
    """Each special-value row as its own tensor, so the NVFP4 tensor scale is
    computed from it (all-zero, -0, subnormal-only, tie-only, ... tensors)."""
    x = edge_tensor()[row:row + 1]
    check_quantize(fp4, orc, x, fmt)


def test_nvfp4_scale_buffer_reused_across_tensors(fp4, orc):
    """The computed s_g never keeps a value from an earlier call through the
    same output word: a large-range tensor, then a small-range one, then an
    all-zero one (s_g = 1), then an empty one (s_g = 1)."""
    import torch
    big = inputs.quant_sweep(rows=8, cols=256, seed=11)
    small = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(big) * np.float32(2.0 ** -20))
    q, s, g = fp4.quantize(to_dev_bf16(big), 1)
    for x in (small, np.zeros_like(big)):
        fp4.quantize(to_dev_bf16(x), 1, out=(q, s, g))
        torch.cuda.synchronize()
        _, _, og = orc.quantize(x, 1)
        assert np.float32(to_np(g)[0]) == np.float32(og)
    empty = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    g.fill_(123.0)
    fp4.quantize(empty, 1, out=(q[:0], s, g))
    torch.cuda.synchronize()
    assert to_np(g)[0] == 1.0


# ------------------------------------------------------------- MSE scales ----
# The "MSE" block-scale method ("FP4 quantization analysis: MXFP4 vs NVFP4"
# §3.2.1, §3.3): the same bit-exact bar as the absmax path.
@pytest.mark.parametrize("shape", [(1, 32), (130, 512), (37, 3104), (5, 32736)])
@pytest.mark.parametrize("fmt", [0, 1])
def test_mse_parity_shapes(fp4, orc, shape, fmt):
    rows, cols = shape
    rng = np.random.default_rng(rows * 5 + cols)
    v = rng.laplace(0, 1, shape).astype(np.float32)
    v[rng.random(shape) < 0.01] *= 20
    check_quantize(fp4, orc, inputs.f32_to_bf16_bits(v), fmt, search=1)


@pytest.mark.parametrize("hk", [16, 32, 64, 128])
@pytest.mark.parametrize("fmt", [0, 1])
def test_mse_parity_rotated(fp4, orc, hk, fmt):
    x = inputs.rotate_acts(rows=136, cols=1024, seed=hk + 1)
    check_quantize(fp4, orc, x, fmt, hk=hk, search=1)


@pytest.mark.parametrize("fmt,tie", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_mse_edge_cases(fp4, orc, fmt, tie):
    """Zeros, -0, subnormals, exact ties, saturation, lone outliers and
    values near the fp32 maximum (whose squared errors overflow to inf on
    both sides, leaving the absmax scale)."""
    x = edge_tensor()
    check_quantize(fp4, orc, x, fmt, tie=tie, search=1)
    check_quantize(fp4, orc, x[:6], fmt, tie=tie, hk=64, search=1)
    for row in range(x.shape[0]):
        check_quantize(fp4, orc, x[row:row + 1], fmt, tie=tie, search=1)


@pytest.mark.parametrize("gscale", [1.0, 1e-3, 1e-30, 3e30])
def test_mse_nvfp4_given_global_scale(fp4, orc, gscale):
    x = inputs.quant_sweep(rows=16, cols=512, seed=13)
    check_quantize(fp4, orc, x, 1, gscale=gscale, search=1)
    check_quantize(fp4, orc, x, 1, gscale=gscale, search=1, tie=1)


@pytest.mark.parametrize("fmt", [0, 1])
def test_mse_full_size_quant_sweep(fp4, orc, fmt):
    """1024 x 131072 heavy-tailed tensor, whole-tensor parity, and the
    tensor's error below the absmax method's."""
    import torch
    x = inputs.quant_sweep()
    q, s, g, (oq, os_, og) = check_quantize(fp4, orc, x, fmt, search=1)
    del q, s, g
    torch.cuda.empty_cache()
    xs = x[:64]
    aq, as_, ag = orc.quantize(xs, fmt, gscale=og if fmt else None)
    xf = inputs.bf16_bits_to_f32(xs)
    n_abs = orc.nmse(xf, orc.dequantize(aq, as_, ag, fmt))
    n_mse = orc.nmse(xf, orc.dequantize(oq[:64], os_[:64], og, fmt))
    assert n_mse < n_abs


# ------------------------------------------------ NVFP4 tensor-scale refinement ----
@pytest.mark.parametrize("shape,hk,tie,rounds", [((64, 1024), 0, 0, 1), ((64, 1024), 0, 0, 4), ((37, 3104), 32, 0, 3),
                                                 ((130, 512), 128, 1, 2), ((8, 4096), 16, 0, 5)])
def test_nv_refined_tensor_scale_matches_oracle(fp4, orc, shape, hk, tie, rounds):
    """Alternating MSE-group / least-squares-global refinement ("FP4
    quantization analysis" §3.2.1): the GPU's s_g equals the oracle's bit for
    bit (fixed-order fp64 sums on both sides), and so does the MSE
    quantization under it."""
    import torch
    rows, cols = shape
    x = inputs.f32_to_bf16_bits(inputs.table5_weight(rows * cols, seed=rows + hk).reshape(rows, cols))
    g = fp4.nv_refine_gscale(to_dev_bf16(x), hadamard_k=hk, rounds=rounds, round=tie)
    torch.cuda.synchronize()
    want, _ = orc.nv_refine_gscale(x, hadamard_k=hk, tie=tie, rounds=rounds)
    assert np.float32(to_np(g)[0]) == np.float32(want)
    check_quantize(fp4, orc, x, 1, hk=hk, tie=tie, gscale=want, search=1)


def test_nv_refined_tensor_scale_all_zero(fp4, orc):
    import torch
    g = fp4.nv_refine_gscale(to_dev_bf16(np.zeros((3, 64), np.uint16)), rounds=3)
    torch.cuda.synchronize()
    assert to_np(g)[0] == 1.0
