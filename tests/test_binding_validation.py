"""The Python binding checks every tensor's dtype, shape and layout before it
calls the library: the kernels index all buffers from the sizes of q, so a
smaller k, v, o, dO, LSE or output buffer would be read or written past its
end.  Runs on the CPU: each check fires before the device check and before
any call into the library."""
import pytest
import torch

import exact_io_aware_95_b200 as fa
from exact_io_aware_95_b200 import build as fabuild


@pytest.fixture(scope="module", autouse=True)
def built():
    fabuild.build()


def bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


B, N, H, D = 2, 64, 3, 64


def dense():
    return {"q": bf(B, N, H, D), "k": bf(B, N, H, D), "v": bf(B, N, H, D), "o": bf(B, N, H, D),
            "do": bf(B, N, H, D), "lse": f32(B, H, N)}


@pytest.mark.parametrize("bad", ["k", "v"])
def test_fwd_rejects_mismatched_inputs(bad):
    x = dense()
    x[bad] = bf(B, N - 1, H, D)
    with pytest.raises(ValueError):
        fa.fwd(x["q"], x["k"], x["v"])


@pytest.mark.parametrize("which,shape,dtype", [("out", (B, N, H, D - 1), torch.bfloat16),
                                               ("out", (B, N, H, D), torch.float32),
                                               ("lse", (B, N, H), torch.float32),
                                               ("lse", (B, H, N - 1), torch.float32)])
def test_fwd_rejects_bad_outputs(which, shape, dtype):
    x = dense()
    kw = {which: torch.zeros(*shape, dtype=dtype)}
    with pytest.raises((ValueError, TypeError)):
        fa.fwd(x["q"], x["k"], x["v"], **kw)


@pytest.mark.parametrize("bad", ["k", "v", "o", "do"])
def test_bwd_rejects_mismatched_inputs(bad):
    x = dense()
    x[bad] = bf(B, N, H - 1, D)
    with pytest.raises(ValueError):
        fa.bwd(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"])


def test_bwd_rejects_bad_lse():
    x = dense()
    with pytest.raises(ValueError):
        fa.bwd(x["q"], x["k"], x["v"], x["o"], f32(B, H, N // 2), x["do"])


@pytest.mark.parametrize("which", ["dq", "dk", "dv"])
def test_bwd_rejects_bad_gradient_buffers(which):
    x = dense()
    with pytest.raises(ValueError):
        fa.bwd(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"], **{which: bf(B, N, H, D // 2)})
    with pytest.raises(TypeError):
        fa.bwd(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"], **{which: f32(B, N, H, D)})
    with pytest.raises(ValueError):  # non-contiguous
        fa.bwd(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"], **{which: bf(B, H, N, D).transpose(1, 2)})


def test_bwd_rejects_small_workspace():
    x = dense()
    ws = torch.zeros(fa.workspace_size(B, N, H, D) - 16, dtype=torch.uint8)
    with pytest.raises(fa.FaError) as e:
        fa.bwd(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"], workspace=ws)
    assert e.value.status == fa.FA_ERR_WORKSPACE


def test_varlen_rejects_mismatched_shapes():
    T = 100
    q, k, v, o, do = (bf(T, H, D) for _ in range(5))
    cu = torch.tensor([0, 40, 100], dtype=torch.int32)
    with pytest.raises(ValueError):
        fa.varlen_fwd(q, bf(T - 1, H, D), v, cu, 60)
    with pytest.raises(ValueError):
        fa.varlen_fwd(q, k, v, cu, 60, lse=f32(H, T + 1))
    with pytest.raises(ValueError):
        fa.varlen_bwd(q, k, v, o, f32(H, T - 1), do, cu, 60)
    with pytest.raises(ValueError):
        fa.varlen_bwd(q, k, v, bf(T, H, D // 2), f32(H, T), do, cu, 60)
    with pytest.raises(ValueError):
        fa.varlen_bwd(q, k, v, o, f32(H, T), do, cu, 60, dq=bf(T - 1, H, D))


def test_decode_rejects_bad_outputs():
    q = bf(2, 1, H, D)
    kc = bf(2, 300, H, D)
    with pytest.raises(ValueError):
        fa.decode_fwd(q, kc, kc, out=bf(2, 2, H, D))
    with pytest.raises(ValueError):
        fa.decode_fwd(q, kc, kc, lse=f32(2, 1, H))


def test_cpu_tensors_are_refused_after_the_shape_checks():
    x = dense()
    with pytest.raises(ValueError, match="CUDA device"):
        fa.fwd(x["q"], x["k"], x["v"])
