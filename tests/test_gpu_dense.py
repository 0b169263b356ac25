"""The dense-decoder variant (n_experts = 0: no router, one SwiGLU FFN per
layer held as the shared expert) against the CPU oracle, through the C ABI."""
import pytest
import torch

from synthetic import ModelConfig, Workload, workload

from parity import Session, run_greedy

pytestmark = pytest.mark.gpu

# off the tile grid: d not a multiple of 256, FFN not a multiple of 256, hd 64
RAGGED_DENSE = ModelConfig("ragged_dense", n_layers=2, d_model=264, n_q_heads=6, n_kv_heads=2,
                           head_dim=64, n_experts=0, top_k=0, expert_ffn=16, shared_ffn=80,
                           vocab=1000, sigma=0.05)
# mid-size: the small model's attention with a 5632-wide FFN
MID_DENSE = ModelConfig("mid_dense", n_layers=4, d_model=2048, n_q_heads=16, n_kv_heads=4,
                        head_dim=128, n_experts=0, top_k=0, expert_ffn=16, shared_ffn=5632,
                        vocab=32000)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


@pytest.mark.parametrize("variant", ["megakernel", "multikernel"])
def test_tiny_dense_greedy(variant):
    s = Session(workload("tiny_dense"), variant=variant)
    rep = run_greedy(s, 16)
    s.close()
    assert rep.argmax_checked >= 14 and rep.expert_near_ties == 0  # no router: empty expert sets
    print(variant, rep)


@pytest.mark.parametrize("B", [1, 3, 8])
def test_ragged_dense(B):
    wl = Workload(f"ragged_dense_b{B}", RAGGED_DENSE, B, 1, context=None, context_range=(1, 70),
                  steps=4, seed=9)
    s = Session(wl, capacity=96)
    rep = run_greedy(s, 4)
    s.close()
    print(B, rep)


@pytest.mark.parametrize("B", [1, 2])
def test_mid_dense(B):
    wl = Workload(f"mid_dense_b{B}", MID_DENSE, B, 1, context=None, context_range=(700, 1500),
                  steps=3, seed=10)
    s = Session(wl)
    rep = run_greedy(s, 3)
    s.close()
    assert rep.argmax_checked >= 2
    print(B, rep)


def test_dense_full_size():
    """The benchmark's dense workload at full size (16 layers, d 4096, a
    14336-wide FFN, vocab 64000; about 8 GB of weights), two whole steps; the
    oracle fetches each layer's weights from the device."""
    s = Session(workload("dense", 1), cache_host_weights=False)
    rep = run_greedy(s, 2)
    s.close()
    assert rep.argmax_checked >= 1
    print(rep)
