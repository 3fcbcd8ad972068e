"""Shared helpers of the GPU parity tests: move a workload to the device, run one
decode step through the library, compare with the oracle."""
import numpy as np

ATOL_MAX = 1e-2   # max-abs error bound for attention outputs vs the fp64 oracle
ATOL_MEAN = 1e-3  # mean-abs error bound


def bf16_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def i32_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def bits_host(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class DeviceCase:
    def __init__(self, case):
        import torch
        self.case = case
        self.q = bf16_dev(case.q)
        self.k = bf16_dev(case.k_cache)
        self.v = bf16_dev(case.v_cache)
        self.k_new = bf16_dev(case.k_new)
        self.v_new = bf16_dev(case.v_new)
        self.slots = i32_dev(case.slot_mapping)
        self.pairs = i32_dev(case.copy_pairs.reshape(-1, 2))
        self.tables = i32_dev(case.block_tables)
        self.lens = i32_dev(case.seq_lens)
        self.out = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
        self.flag = torch.zeros(1, dtype=torch.int32, device="cuda")


def run_step(dc, partition_tokens=None, tables=None, k=None, v=None):
    """copy_blocks -> reshape_and_cache -> decode, as one decode step."""
    import torch
    import paged_kv_cache_349_b200 as pa
    c = dc.case
    k = dc.k if k is None else k
    v = dc.v if v is None else v
    tables = dc.tables if tables is None else tables
    pt = c.partition_tokens if partition_tokens is None else partition_tokens
    pa.pa_copy_blocks(k, v, dc.pairs, err_flag=dc.flag)
    pa.pa_reshape_and_cache(dc.k_new, dc.v_new, k, v, dc.slots, err_flag=dc.flag)
    ws_bytes = pa.pa_decode_workspace_size(c.batch, c.num_q_heads, c.num_kv_heads, c.head_dim,
                                           c.block_size, c.max_seq_len, pt)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda") if ws_bytes else None
    pa.pa_decode(dc.out, dc.q, k, v, tables, dc.lens, max_seq_len=c.max_seq_len,
                 scale=float(c.scale), partition_tokens=pt, workspace=ws, err_flag=dc.flag)
    torch.cuda.synchronize()
    return dc.out.cpu().numpy().astype(np.float64)


def assert_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, what
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    assert err.max() <= ATOL_MAX, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= ATOL_MEAN, f"{what}: mean-abs {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def sample_rows(case, n, seed=0):
    rng = np.random.default_rng(seed)
    b = rng.integers(0, case.batch, size=n)
    g = rng.integers(0, case.num_q_heads, size=n)
    # always include the longest and the shortest sequence
    b[0] = int(np.argmax(case.seq_lens))
    b[1] = int(np.argmin(case.seq_lens))
    return np.stack([b, g], axis=1).astype(np.int32)


def run_fused_step(dc, partition_tokens=None):
    """copy_blocks -> (cache write of tokens other than each sequence's last) -> pa_decode_append."""
    import torch
    import paged_kv_cache_349_b200 as pa
    c = dc.case
    pt = c.partition_tokens if partition_tokens is None else partition_tokens
    import workloads as W
    k_last, v_last, other = W.split_last_tokens(c)
    pa.pa_copy_blocks(dc.k, dc.v, dc.pairs, err_flag=dc.flag)
    if other.size:
        pa.pa_reshape_and_cache(bf16_dev(c.k_new[other]), bf16_dev(c.v_new[other]), dc.k, dc.v,
                                i32_dev(c.slot_mapping[other]), err_flag=dc.flag)
    ws_bytes = pa.pa_decode_workspace_size(c.batch, c.num_q_heads, c.num_kv_heads, c.head_dim,
                                           c.block_size, c.max_seq_len, pt)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda") if ws_bytes else None
    pa.pa_decode_append(dc.out, dc.q, bf16_dev(k_last), bf16_dev(v_last), dc.k, dc.v, dc.tables, dc.lens,
                        max_seq_len=c.max_seq_len, scale=float(c.scale), partition_tokens=pt, workspace=ws,
                        err_flag=dc.flag)
    torch.cuda.synchronize()
    return dc.out.cpu().numpy().astype(np.float64)
