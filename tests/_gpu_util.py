"""Helpers shared by the GPU parity tests (not collected as tests)."""
import numpy as np
import torch

import oracle
import paged_kv_cache_420_b200 as pkv

# Attention tolerance of the parity bar: max-abs error and relative L2 error of
# the whole output tensor against the fp64 oracle.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def to_cuda(w):
    """Moves a workload's tensors to cuda:0 (in place) and returns it."""
    for name in ("q", "k_new", "v_new", "k_cache", "v_cache"):
        setattr(w, name, getattr(w, name).to("cuda").contiguous())
    return w


def device_inputs(w):
    return dict(
        slots=torch.from_numpy(w.slot_mapping).to("cuda"),
        tables=torch.from_numpy(w.block_tables).to("cuda"),
        ctx=torch.from_numpy(w.context_lens).to("cuda"),
    )


def run_step(w, partition_tokens=None, kc=None, vc=None, attention=True):
    """Copy-on-write pairs, slot-mapped write and decode attention through the
    library, on copies of the workload's pools.  Returns (kc, vc, out)."""
    kc = w.k_cache.clone() if kc is None else kc
    vc = w.v_cache.clone() if vc is None else vc
    d = device_inputs(w)
    if len(w.copy_pairs):
        pkv.pkv_copy_blocks(w.copy_pairs, kc, vc)
    pkv.pkv_write(w.k_new, w.v_new, d["slots"], kc, vc)
    out = None
    if attention:
        out = torch.empty_like(w.q)
        pt = w.partition_tokens if partition_tokens is None else partition_tokens
        pkv.paged_attn_decode(w.q, kc, vc, d["tables"], d["ctx"], w.scale, w.num_kv_heads, out,
                              max_context_len=w.max_context_len, partition_tokens=pt)
    torch.cuda.synchronize()
    return kc, vc, out


def bits_equal(gpu_bf16: torch.Tensor, oracle_bits: np.ndarray) -> bool:
    g = gpu_bf16.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return g.shape == oracle_bits.shape and np.array_equal(g, oracle_bits)


def attention_errors(out_gpu: torch.Tensor, ref: np.ndarray):
    got = out_gpu.float().cpu().double().numpy()
    err = got - ref
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    return max_abs, rel


def assert_attention_close(out_gpu, ref, what=""):
    got = out_gpu.float().cpu().numpy()
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    max_abs, rel = attention_errors(out_gpu, ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def no_device_error():
    code = pkv.get_device_error()
    assert code == 0, f"device error word {code:#x}"
