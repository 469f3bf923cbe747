"""The Python binding rejects malformed tensors before anything reaches a
kernel (needs a CUDA device: the checks run on CUDA tensors).  A short
codebook or a wrong-sized output would otherwise be read or written out of
bounds on the device."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import differentiable_bcjr_b200 as B
    B.lib()
    return B


def _t(*shape, dtype=torch.float32):
    return torch.zeros(shape, dtype=dtype, device="cuda")


def test_bitshift_calls_check_their_tensors(B):
    w, c = _t(3, 8), _t(256)
    with pytest.raises(ValueError):
        B.bcjr_forward(w, _t(255), 0.5, 8, 2)                 # short codebook
    with pytest.raises(ValueError):
        B.bcjr_forward(w, c, 0.5, 8, 2, out=_t(3, 7))         # wrong output shape
    with pytest.raises(ValueError):
        B.bcjr_forward(w.double(), c, 0.5, 8, 2)              # not float32
    with pytest.raises(ValueError):
        B.bcjr_forward(_t(24), c, 0.5, 8, 2)                  # not [n_seq][seq_len]
    with pytest.raises(ValueError):
        B.bcjr_backward(w, w, c, w, 0.5, 8, 2, grad_codebook=_t(128))
    with pytest.raises(ValueError):
        B.bcjr_backward(_t(3, 9), w, c, w, 0.5, 8, 2)
    with pytest.raises(ValueError):
        B.viterbi_decode(w, _t(64), 8, 2)


def test_dense_calls_check_their_tensors(B):
    w, c, lam = _t(3, 8), _t(256), _t(256, 256)
    with pytest.raises(ValueError):
        B.bcjr_dense_forward(w, c, _t(256, 255), 0.5)
    with pytest.raises(ValueError):
        B.bcjr_dense_backward(w, w, c, lam, _t(3, 7), 0.5)
    with pytest.raises(ValueError):
        B.bcjr_dense_backward(w, w, c, lam, w, 0.5, want_grad_log_trans=True, grad_log_trans=_t(256))
