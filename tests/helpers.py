"""Test-only helpers: bf16 bit conversion and small brute-force references."""
import numpy as np


def f32_to_bf16_bits(x):
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f64(h):
    u = np.asarray(h, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def ulp32(x):
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(x).astype(np.float64)


def sub_problem(inp, wl, b, kvh):
    """(sequence b, kv head kvh) of a device workload as a self-contained host
    problem for the oracle: that kv head's pages in logical order (identity
    page table), the group's queries, and the physical blocks they came from."""
    from sparse_entmax_kv_b200.workloads import to_host_u16
    L = int(inp["seq_lens"][b])
    npb = -(-L // wl.P)
    blocks = inp["page_table"][b, :npb].long()
    G = wl.G
    K = inp["k_cache"][blocks, kvh:kvh + 1].contiguous()
    V = inp["v_cache"][blocks, kvh:kvh + 1].contiguous()
    q = inp["q"][b:b + 1, kvh * G:(kvh + 1) * G].contiguous()
    return dict(q=to_host_u16(q), K=to_host_u16(K), V=to_host_u16(V),
                page_table=np.arange(npb, dtype=np.int32)[None], seq_lens=np.array([L], np.int32), npb=npb,
                blocks=blocks.cpu().numpy())
