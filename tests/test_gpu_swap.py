"""pa_swap_blocks: device <-> pinned host block swaps, bit-exact against the oracle."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import bf16_dev, bits_host, i32_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch


@pytest.mark.parametrize("d,bs", [(128, 16), (64, 32)])
def test_swap_out_and_back_in(torch_cuda, d, bs):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    rng = np.random.default_rng(d + bs)
    NBd, NBh, Hkv = 96, 40, 4
    dev_k = W.bf16_normal(rng, (NBd, Hkv, bs, d))
    dev_v = W.bf16_normal(rng, (NBd, Hkv, bs, d))
    host_k = np.full((NBh, Hkv, bs, d), W.BF16_QNAN, np.uint16)
    host_v = host_k.copy()
    out_pairs = np.stack([rng.choice(NBd, 30, replace=False), rng.choice(NBh, 30, replace=False)], 1).astype(np.int32)
    in_pairs = np.stack([out_pairs[:, 1], rng.choice(NBd, 30, replace=False)], 1).astype(np.int32)

    # oracle: out to host, then back into other device blocks
    o_hk, o_hv = host_k.copy(), host_v.copy()
    o_dk, o_dv = dev_k.copy(), dev_v.copy()
    assert oracle.swap_blocks(o_hk, o_hv, o_dk, o_dv, out_pairs) == 0
    assert oracle.swap_blocks(o_dk, o_dv, o_hk, o_hv, in_pairs) == 0

    g_dk, g_dv = bf16_dev(dev_k), bf16_dev(dev_v)
    g_hk = torch.from_numpy(host_k.view(np.int16)).view(torch.bfloat16).pin_memory()
    g_hv = torch.from_numpy(host_v.view(np.int16)).view(torch.bfloat16).pin_memory()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_swap_blocks(g_hk, g_hv, g_dk, g_dv, i32_dev(out_pairs), err_flag=flag)      # swap-out
    pa.pa_swap_blocks(g_dk, g_dv, g_hk, g_hv, i32_dev(in_pairs), err_flag=flag)       # swap-in
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    assert np.array_equal(g_hk.view(torch.int16).numpy().view(np.uint16), o_hk)
    assert np.array_equal(g_hv.view(torch.int16).numpy().view(np.uint16), o_hv)
    assert np.array_equal(bits_host(g_dk), o_dk) and np.array_equal(bits_host(g_dv), o_dv)


def test_swap_bad_pair_flagged(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    k = torch.zeros((4, 1, 16, 64), dtype=torch.bfloat16, device="cuda")
    h = torch.ones((2, 1, 16, 64), dtype=torch.bfloat16).pin_memory()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_swap_blocks(k, k, h, h, i32_dev(np.array([[2, 0], [1, 3]], np.int32)), err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == pa.PA_FLAG_BAD_PAIR
    assert float(k[3].float().sum()) == 16 * 64 and float(k[0].float().sum()) == 0


def test_swap_rejects_pageable_host_memory(torch_cuda):
    """A host pool the device cannot address (pageable memory) is an argument error caught before any
    launch: nothing is copied and the flag stays clear."""
    import ctypes
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    k = torch.ones((4, 1, 16, 64), dtype=torch.bfloat16, device="cuda")
    pageable = np.zeros((4, 1, 16, 64), np.uint16)           # plain numpy memory, never registered with CUDA
    pairs = i32_dev(np.array([[0, 1]], np.int32))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    hp = ctypes.c_void_p(pageable.ctypes.data)
    dp = ctypes.c_void_p(k.data_ptr())
    before = pa.launch_count()
    rc = lib.pa_swap_blocks(hp, hp, 4, dp, dp, 4, ctypes.c_void_p(pairs.data_ptr()), 1, 1, 16, 64,
                            ctypes.c_void_p(flag.data_ptr()), None)
    assert rc == pa.PA_ERR_INVALID_ARG
    rc = lib.pa_swap_blocks(dp, dp, 4, hp, hp, 4, ctypes.c_void_p(pairs.data_ptr()), 1, 1, 16, 64,
                            ctypes.c_void_p(flag.data_ptr()), None)
    assert rc == pa.PA_ERR_INVALID_ARG
    # pairs in pageable host memory too
    hpairs = np.array([[0, 1]], np.int32)
    rc = lib.pa_swap_blocks(dp, dp, 4, dp, dp, 4, ctypes.c_void_p(hpairs.ctypes.data), 1, 1, 16, 64,
                            ctypes.c_void_p(flag.data_ptr()), None)
    assert rc == pa.PA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert pa.launch_count() == before
    assert int(flag.item()) == 0 and not pageable.any() and float(k.float().sum()) == 4 * 16 * 64
