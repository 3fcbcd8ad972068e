"""pa_decode_append (cache write fused into decode) vs the oracle and vs the unfused step."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import DeviceCase, assert_close, bits_host, run_fused_step, run_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _check(case, pt=None, what=""):
    fused = DeviceCase(case)
    got = run_fused_step(fused, pt)
    want, k_ref, v_ref = oracle.decode_step(case)
    assert np.array_equal(bits_host(fused.k), k_ref), f"{what}: K pool differs"
    assert np.array_equal(bits_host(fused.v), v_ref), f"{what}: V pool differs"
    assert int(fused.flag.item()) == 0
    assert_close(got, want, what)
    unfused = DeviceCase(case)
    ref = run_step(unfused, pt)
    assert np.array_equal(got, ref), f"{what}: fused and unfused outputs differ"


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (2, dict(batch=6, max_len=300, num_blocks=256)),
    (3, dict(batch=8, max_len=260, num_blocks=512)),
    (4, dict(batch=9, max_len=700, num_blocks=256)),
    (5, dict(batch=2, max_len=2048, num_blocks=640, num_copy_pairs=40)),
])
def test_workloads(cfg, kw):
    _check(W.make_case(cfg, **kw), what=f"cfg{cfg}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_ragged_shapes(d, bs, G):
    lens = [0, 1, 2, 15, 16, 17, 31, 32, 33, 48, 49, 257]
    case = W.make_custom_case(lens, num_q_heads=2 * G, num_kv_heads=2, head_dim=d, block_size=bs,
                              seed=100 + d + bs + G)
    for pt in (-1, bs, 2 * bs):
        _check(case, pt, what=f"d{d} bs{bs} G{G} pt{pt}")


def test_full_size_llama2_7b_sampled_rows():
    from tests.gpu_helpers import sample_rows
    case = W.make_case(2)
    dc = DeviceCase(case)
    got = run_fused_step(dc)
    rows = sample_rows(case, 64, seed=9)
    want, k_ref, v_ref = oracle.decode_step(case, rows=rows)
    assert np.array_equal(bits_host(dc.k), k_ref) and np.array_equal(bits_host(dc.v), v_ref)
    assert_close(got[rows[:, 0], rows[:, 1]], want, "cfg2 full fused")
