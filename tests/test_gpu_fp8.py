"""fp8 (E4M3) pools on the GPU against the fp64 oracle.

Quantised codes (bulk conversion and cache write) must be bit-exact with the
oracle's encoder; decode over fp8 pools must match the oracle's attention on
the dequantised rows within the attention tolerance; the fused write must
match the two-launch path bit for bit; copy and swap move bytes exactly.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import assert_close, bf16_dev, i32_dev, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch


def u8_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def u8_host(t):
    return t.cpu().numpy()


def amax_scale(bits):
    vals = bits.view(np.uint16).astype(np.uint32) << 16
    f = vals.view(np.float32)
    f = f[np.isfinite(f)]
    return float(np.abs(f).max() / 448.0) if f.size else 1.0


def test_quantize_matches_oracle(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    rng = np.random.default_rng(3)
    x = W.bf16_normal(rng, (4096,))
    # plus hand-picked values: ties, saturation, subnormal range, zeros, NaN
    extra = np.array([1.0625, 1.1875, 449.0, -449.0, 1e6, 2 ** -9, 3 * 2 ** -10, 0.0, -0.0, 240.0, 30.0, 2 ** -12],
                     np.float32)
    x = np.concatenate([x, W.bf16_bits(extra), np.array([0x7FC0, 0x0000, 0x8000, 0x0001], np.uint16)])
    x = np.concatenate([x, np.zeros((-x.size) % 8, np.uint16)])
    for scale in (1.0, 0.1, 3.0 / 448.0, 1e-3):
        dst = torch.empty(x.size, dtype=torch.uint8, device="cuda")
        pa.pa_quantize_fp8(bf16_dev(x), dst, scale)
        torch.cuda.synchronize()
        assert np.array_equal(u8_host(dst), oracle.quantize_e4m3(x, scale)), scale


def _fp8_case(case, k_scale, v_scale):
    """fp8 pools (oracle-quantised) holding the case's cached tokens."""
    return oracle.quantize_e4m3(case.k_cache, k_scale), oracle.quantize_e4m3(case.v_cache, v_scale)


def _oracle_step_fp8(case, k8, v8, k_scale, v_scale, rows=None):
    k8, v8 = k8.copy(), v8.copy()
    # block copies move bytes (the oracle's copy on a 16-bit view of the same bytes),
    # the write quantises, decode reads dequantised rows
    assert oracle.copy_blocks(k8.view(np.uint16), v8.view(np.uint16), case.copy_pairs) == 0
    assert oracle.reshape_and_cache_fp8(case.k_new, case.v_new, k8, v8, case.slot_mapping, case.block_size,
                                        k_scale, v_scale) == 0
    out = oracle.decode_fp8(case.q, k8, v8, case.block_tables, case.seq_lens, num_kv_heads=case.num_kv_heads,
                            block_size=case.block_size, scale=case.scale, k_scale=k_scale, v_scale=v_scale,
                            rows=rows)
    return out, k8, v8


def _gpu_step_fp8(case, k8, v8, k_scale, v_scale, pt=None, fused=False):
    import torch
    import paged_kv_cache_349_b200 as pa
    pt = case.partition_tokens if pt is None else pt
    gk, gv = u8_dev(k8), u8_dev(v8)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks_fp8(gk, gv, i32_dev(case.copy_pairs.reshape(-1, 2)), err_flag=flag)
    out = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
    ws_b = pa.pa_decode_workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                       case.block_size, case.max_seq_len, pt)
    ws = torch.empty(max(ws_b, 16), dtype=torch.uint8, device="cuda")
    kw = dict(max_seq_len=case.max_seq_len, scale=float(case.scale), k_scale=k_scale, v_scale=v_scale,
              partition_tokens=pt, workspace=ws, err_flag=flag)
    if fused:
        k_last, v_last, other = W.split_last_tokens(case)
        if other.size:
            pa.pa_reshape_and_cache_fp8(bf16_dev(case.k_new[other]), bf16_dev(case.v_new[other]), gk, gv,
                                        i32_dev(case.slot_mapping[other]), k_scale=k_scale, v_scale=v_scale,
                                        err_flag=flag)
        pa.pa_decode_fp8(out, bf16_dev(case.q), gk, gv, i32_dev(case.block_tables), i32_dev(case.seq_lens),
                         k_new=bf16_dev(k_last), v_new=bf16_dev(v_last), **kw)
    else:
        pa.pa_reshape_and_cache_fp8(bf16_dev(case.k_new), bf16_dev(case.v_new), gk, gv, i32_dev(case.slot_mapping),
                                    k_scale=k_scale, v_scale=v_scale, err_flag=flag)
        pa.pa_decode_fp8(out, bf16_dev(case.q), gk, gv, i32_dev(case.block_tables), i32_dev(case.seq_lens), **kw)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    return out.cpu().numpy().astype(np.float64), u8_host(gk), u8_host(gv)


def _check(case, pt=None, what=""):
    k_scale = amax_scale(case.k_cache)
    v_scale = amax_scale(case.v_cache) / 2      # some values saturate
    k8, v8 = _fp8_case(case, k_scale, v_scale)
    want, k_ref, v_ref = _oracle_step_fp8(case, k8, v8, k_scale, v_scale)
    got, gk, gv = _gpu_step_fp8(case, k8, v8, k_scale, v_scale, pt)
    assert np.array_equal(gk, k_ref) and np.array_equal(gv, v_ref), f"{what}: fp8 pools differ"
    assert_close(got, want, what)
    fused, fk, fv = _gpu_step_fp8(case, k8, v8, k_scale, v_scale, pt, fused=True)
    assert np.array_equal(fk, k_ref) and np.array_equal(fv, v_ref), f"{what}: fused fp8 pools differ"
    assert np.array_equal(fused, got), f"{what}: fused and unfused fp8 outputs differ"


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (2, dict(batch=6, max_len=300, num_blocks=256)),
    (3, dict(batch=8, max_len=260, num_blocks=512)),
    (4, dict(batch=9, max_len=700, num_blocks=256)),
    (5, dict(batch=2, max_len=2048, num_blocks=640, num_copy_pairs=40)),
])
def test_fp8_workloads(torch_cuda, cfg, kw):
    _check(W.make_case(cfg, **kw), what=f"fp8 cfg{cfg}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32, 64])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_fp8_ragged_shapes(torch_cuda, d, bs, G):
    lens = [0, 1, 2, 15, 16, 17, 31, 32, 33, 48, 49, 257]
    case = W.make_custom_case(lens, num_q_heads=2 * G, num_kv_heads=2, head_dim=d, block_size=bs,
                              seed=300 + d + bs + G)
    for pt in (-1, 2 * bs):
        _check(case, pt, what=f"fp8 d{d} bs{bs} G{G} pt{pt}")


def test_fp8_tiny_and_huge_queries(torch_cuda):
    """The power-of-two rescaling of q keeps results right for very small and very large q."""
    case = W.make_case(2, batch=3, max_len=200, num_blocks=64)
    for factor in (2.0 ** -60, 2.0 ** 40):
        vals = (case.q.astype(np.uint32) << 16).view(np.float32) * np.float32(factor)
        case.q = W.bf16_bits(vals)
        _check(case, -1, what=f"q x {factor}")
        case.q = W.bf16_bits((case.q.astype(np.uint32) << 16).view(np.float32) / np.float32(factor))


def test_fp8_swap_and_copy_bytes(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    rng = np.random.default_rng(5)
    dev = rng.integers(0, 256, size=(64, 2, 16, 128), dtype=np.uint8)
    host = np.zeros((32, 2, 16, 128), np.uint8)
    pairs = np.stack([rng.choice(64, 20, replace=False), rng.choice(32, 20, replace=False)], 1).astype(np.int32)
    gk, gv = u8_dev(dev), u8_dev(dev[::-1].copy())
    hk = torch.from_numpy(host.copy()).pin_memory()
    hv = torch.from_numpy(host.copy()).pin_memory()
    pa.pa_swap_blocks_fp8(hk, hv, gk, gv, i32_dev(pairs))
    cp = np.stack([rng.choice(32, 10, replace=False), 32 + rng.choice(32, 10, replace=False)], 1).astype(np.int32)
    pa.pa_copy_blocks_fp8(gk, gv, i32_dev(cp))
    torch.cuda.synchronize()
    want_h = host.copy()
    want_h[pairs[:, 1]] = dev[pairs[:, 0]]
    assert np.array_equal(hk.numpy(), want_h)
    want_d = dev.copy()
    want_d[cp[:, 1]] = dev[cp[:, 0]]
    assert np.array_equal(u8_host(gk), want_d)


def test_fp8_full_size_llama2_7b_sampled_rows(torch_cuda):
    case = W.make_case(2)
    k_scale, v_scale = amax_scale(case.k_cache), amax_scale(case.v_cache)
    k8, v8 = _fp8_case(case, k_scale, v_scale)
    rows = sample_rows(case, 48, seed=12)
    want, k_ref, v_ref = _oracle_step_fp8(case, k8, v8, k_scale, v_scale, rows=rows)
    got, gk, gv = _gpu_step_fp8(case, k8, v8, k_scale, v_scale, fused=True)
    assert np.array_equal(gk, k_ref) and np.array_equal(gv, v_ref)
    assert_close(got[rows[:, 0], rows[:, 1]], want, "fp8 cfg2 full")


@pytest.mark.parametrize("cfg,kw,chunks", [
    (2, dict(batch=64, max_len=300, num_blocks=2048), 0),
    (2, dict(batch=6, max_len=300, num_blocks=256), 1),
    (4, dict(batch=9, max_len=1500, num_blocks=512), 4),                              # split decode
    (5, dict(batch=3, max_len=2048, num_blocks=960, num_copy_pairs=40), 3),           # E4M3 block copies
])
def test_fp8_host_step_matches_device_path(torch_cuda, cfg, kw, chunks):
    """pa_decode_step_host_fp8 == fp8 block copies + fused fp8 write and decode on the device, bit for bit."""
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    case = W.make_case(cfg, **kw)
    k_last, v_last, other = W.split_last_tokens(case)
    assert other.size == 0
    k_scale, v_scale = amax_scale(case.k_cache), amax_scale(case.v_cache)
    k8, v8 = _fp8_case(case, k_scale, v_scale)
    want, want_k, want_v = _gpu_step_fp8(case, k8, v8, k_scale, v_scale, fused=True)

    def pinned(a, dtype):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(dtype) if dtype is torch.bfloat16 else t.to(dtype)).pin_memory()

    pairs = case.copy_pairs.reshape(-1, 2)
    max_pairs = max(1, pairs.shape[0])
    pairs_np = np.zeros((max_pairs, 2), np.int32)
    pairs_np[:pairs.shape[0]] = pairs
    out_h = torch.full(case.q.shape, float("nan"), dtype=torch.float32).pin_memory()
    gk, gv = u8_dev(k8), u8_dev(v8)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    size = pa.pa_decode_step_staging_size(case.batch, case.max_blocks_per_seq, max_pairs, case.num_q_heads,
                                          case.num_kv_heads, case.head_dim, case.block_size, case.max_seq_len,
                                          case.partition_tokens)
    staging = torch.empty(size, dtype=torch.uint8, device="cuda")
    step = pa.DecodeStepHost(out_host=out_h, q_host=pinned(case.q.view(np.int16), torch.bfloat16),
                             k_new_host=pinned(k_last.view(np.int16), torch.bfloat16),
                             v_new_host=pinned(v_last.view(np.int16), torch.bfloat16),
                             tables_host=pinned(case.block_tables, torch.int32),
                             lens_host=pinned(case.seq_lens, torch.int32), pairs_host=pinned(pairs_np, torch.int32),
                             k_cache=gk, v_cache=gv, scale=float(case.scale), k_scale=k_scale, v_scale=v_scale,
                             max_seq_len_cap=case.max_seq_len,
                             partition_tokens=case.partition_tokens, num_chunks=chunks, staging=staging,
                             err_flag=flag)
    step(case.max_seq_len, pairs.shape[0])
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    assert np.array_equal(out_h.numpy().astype(np.float64), want)
    assert np.array_equal(u8_host(gk), want_k) and np.array_equal(u8_host(gv), want_v)

