"""Host-side argument checks of the Python binding (no GPU needed): the library
reads raw pointers, so the binding rejects buffers of the wrong size or type
before anything is enqueued."""
import pytest
import torch

from sub_quadratic_attention_b200 import binding as b


def _args(B=2, L=64, H=2, D=4, dtype=torch.bfloat16, nb=None, complex_gate=False):
    C = H * D
    nb = L // 2 + 1 if nb is None else nb
    tok = [torch.zeros(B, L, C, dtype=dtype) for _ in range(5)]   # q, k, v, x, y
    G = torch.zeros(H, nb, dtype=torch.complex64 if complex_gate else torch.float32)
    return dict(q=tok[0], k=tok[1], v=tok[2], x=tok[3], G=G, gamma=torch.ones(C),
                beta=torch.zeros(C), y=tok[4])


def _check(a, B=2, L=64, H=2, D=4, plan_L=None, code=None, out=None):
    code = b.SPECTRE_BF16 if code is None else code
    b.check_arguments(B, L, H, H * D, L if plan_L is None else plan_L, code, a["q"], a["k"],
                      a["v"], a["x"], a["G"], a["gamma"], a["beta"], a["y"], out)


def test_valid_arguments_pass():
    _check(_args())
    _check(_args(dtype=torch.float32), code=b.SPECTRE_F32, out=torch.zeros(2, 64, 8))
    _check(_args(complex_gate=True))
    _check(_args(nb=9), plan_L=16)             # blockwise: the gate is the block's


@pytest.mark.parametrize("field,bad", [
    ("q", torch.zeros(2, 63, 8, dtype=torch.bfloat16)),
    ("x", torch.zeros(2, 64, 8, dtype=torch.float32)),      # plan is bf16
    ("y", torch.zeros(2, 64, 7, dtype=torch.bfloat16)),
    ("G", torch.zeros(2, 32)),
    ("G", torch.zeros(2, 33, dtype=torch.bfloat16)),
    ("gamma", torch.ones(7)),
    ("beta", torch.zeros(8, dtype=torch.float64)),
])
def test_wrong_size_or_type_is_rejected(field, bad):
    a = _args()
    a[field] = bad
    with pytest.raises(ValueError):
        _check(a)


def test_full_length_gate_is_rejected_in_block_mode():
    with pytest.raises(ValueError):
        _check(_args(), plan_L=16)


def test_wrong_debug_output_is_rejected():
    with pytest.raises(ValueError):
        _check(_args(), out=torch.zeros(2, 64, 8, dtype=torch.bfloat16))


@pytest.mark.parametrize("block_len", [0, -4, 48, 100])
def test_block_len_must_divide_L(block_len):
    with pytest.raises(ValueError):
        b.SpectreMix(1, 64, 1, 16, block_len=block_len)


def _dct_args(T=5, d=64, dtype=torch.bfloat16):
    return dict(x=torch.zeros(T, d, dtype=dtype), w=torch.ones(d), gamma=torch.ones(d),
                beta=torch.zeros(d), y=torch.zeros(T, d, dtype=dtype),
                H=torch.zeros(T), route=torch.zeros(T, dtype=torch.uint8))


def test_dct_arguments_return_the_row_count():
    a = _dct_args()
    assert b.check_dct_arguments(64, b.SPECTRE_BF16, **a) == 5
    a = _dct_args(T=0, dtype=torch.float32)
    assert b.check_dct_arguments(64, b.SPECTRE_F32, **a, mix=torch.zeros(0, 64)) == 0


@pytest.mark.parametrize("field,bad", [
    ("x", torch.zeros(5, 63, dtype=torch.bfloat16)),
    ("y", torch.zeros(5, 64, dtype=torch.float32)),
    ("w", torch.ones(32)),
    ("gamma", torch.ones(64, dtype=torch.float64)),
    ("H", torch.zeros(4)),
    ("route", torch.zeros(5, dtype=torch.bool)),
])
def test_dct_wrong_size_or_type_is_rejected(field, bad):
    a = _dct_args()
    a[field] = bad
    with pytest.raises(ValueError):
        b.check_dct_arguments(64, b.SPECTRE_BF16, **a)
