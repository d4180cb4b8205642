"""GPU parity of the segmented causal-LM loss (segment-based peak cutting) against the
CPU oracle.  Bars: loss within 1e-4 relative (fp32 logits from bf16 operands); the
hidden-state gradient (bf16, formed from bf16 softmax-minus-onehot rows) within
max |gpu - oracle| / rms(oracle) <= 3e-2 with one bf16 ulp of the stored value forgiven;
any segmentation gives the same bits."""
import numpy as np
import pytest
import torch

from oracle import lm_loss as olm
from tests.layer_harness import rel_max_ulp, torch_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import token_sparse_long_b200 as J
    J._lib.load()
    return J


def _case(seed, S, h, V, w_std, n_ignored=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    hid = torch.randn(S, h, generator=g).to(torch.bfloat16)
    w = (torch.randn(V, h, generator=g) * w_std).to(torch.bfloat16)
    lab = torch.randint(0, V, (S,), generator=g, dtype=torch.int32)
    if n_ignored:
        lab[torch.randperm(S, generator=g)[:n_ignored]] = -100
    return hid.cuda(), w.cuda(), lab.cuda()


@pytest.mark.parametrize("S,seg", [(300, 128), (300, 300), (257, 64)])
def test_lm_loss_small(J, S, seg):
    hid, w, lab = _case(1, S, 256, 1024, 0.1, n_ignored=17)
    loss, dh = J.jenga_lm_loss_segmented(hid, w, lab, segment_tokens=seg)
    J.jenga_check_device_status()
    ref_loss, ref_dh = olm.lm_loss(torch_to_f64(hid), torch_to_f64(w), lab.cpu().numpy())
    assert abs(loss.item() - ref_loss) / ref_loss < 1e-4, (loss.item(), ref_loss)
    assert rel_max_ulp(torch_to_f64(dh), ref_dh) < 3e-2
    ign = (lab.cpu().numpy() < 0)
    assert torch_to_f64(dh)[ign].max() == 0 and torch_to_f64(dh)[ign].min() == 0


def test_lm_loss_segmentation_is_bit_identical(J):
    hid, w, lab = _case(2, 700, 512, 2048, 0.05, n_ignored=5)
    l1, d1 = J.jenga_lm_loss_segmented(hid, w, lab, segment_tokens=700)
    l2, d2 = J.jenga_lm_loss_segmented(hid, w, lab, segment_tokens=128)
    l3, d3 = J.jenga_lm_loss_segmented(hid, w, lab, segment_tokens=100)
    assert torch.equal(l1, l2) and torch.equal(l1, l3)
    assert torch.equal(d1, d2) and torch.equal(d1, d3)


def test_lm_loss_all_ignored(J):
    hid, w, lab = _case(3, 200, 128, 512, 0.1)
    lab.fill_(-100)
    loss, dh = J.jenga_lm_loss_segmented(hid, w, lab, segment_tokens=64)
    assert loss.item() == 0.0 and torch.count_nonzero(dh).item() == 0


def test_lm_loss_llama_vocab_sampled_rows(J):
    # Llama-2 output-embedding shape (V 32000, h 4096), ragged segments; full oracle loss and
    # the gradient rows of the segment edges and a random sample
    S, seg = 1024, 384
    hid, w, lab = _case(4, S, 4096, 32000, 0.02, n_ignored=31)
    loss, dh = J.jenga_lm_loss_segmented(hid, w, lab, segment_tokens=seg)
    J.jenga_check_device_status()
    rows = np.unique(np.concatenate([[0, 1, seg - 1, seg, 2 * seg - 1, 2 * seg, S - 1],
                                     np.random.default_rng(0).integers(0, S, 24)]))
    ref_loss, ref_dh = olm.lm_loss(torch_to_f64(hid), torch_to_f64(w), lab.cpu().numpy(), rows=rows)
    assert abs(loss.item() - ref_loss) / ref_loss < 1e-4, (loss.item(), ref_loss)
    assert rel_max_ulp(torch_to_f64(dh)[rows], ref_dh) < 3e-2
