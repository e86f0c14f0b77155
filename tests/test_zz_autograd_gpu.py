"""The autograd wrapper on the GPU (marked gpu): gradients through
torch.autograd equal those of a direct m3_chunked_bwd call with the same
dy, bit for bit (the kernels are deterministic), and the forward returns the
library's outputs."""
import pytest
import torch

from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3
from state_space_lm_b200.autograd import mamba3_scan

pytestmark = pytest.mark.gpu

SCAN = ("x", "dt", "A", "lam", "theta", "B", "C", "D")


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()


@pytest.mark.parametrize("rank", [1, 2])
def test_autograd_equals_direct_backward(rank):
    inp = gen.scan_inputs(2, 100, 2, 64, 128, rank=rank, dtype="bf16", seed=950 + rank, mimo_weights=rank > 1)
    d = {k: v.cuda() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    leaves = {k: d[k].clone().requires_grad_() for k in SCAN}
    kw = dict(W_x=d["Wx"], W_y=d["Wy"]) if rank > 1 else {}
    y, hf, uf, af = mamba3_scan(*[leaves[k] for k in SCAN], 64, **kw)
    dy = gen.grad_seed(inp["x"], 951).cuda()
    (y.float() * dy.float()).sum().backward()
    ref = m3.chunked_bwd(*[d[k] for k in SCAN], dy, 64, **kw)
    fwd = (m3.mimo_chunked_fwd if rank > 1 else m3.siso_chunked_fwd)(*[d[k] for k in SCAN], 64, **kw)
    assert torch.equal(y, fwd[0])
    for k in SCAN:
        assert torch.equal(leaves[k].grad, ref["d" + k].to(leaves[k].dtype)), k
