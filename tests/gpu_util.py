"""Helpers for the GPU tests: move seeded workload arrays to the device and run
the layer through the C ABI (via the package binding).  No layer arithmetic."""
import numpy as np


def to_dev(a, dtype=None):
    import torch
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def layer_to_device(layer):
    import torch
    return dict(
        x=to_dev(layer.x_bits, torch.bfloat16),
        logits=to_dev(layer.logits),
        gu_blocks=to_dev(layer.gate_up.blocks), gu_scales=to_dev(layer.gate_up.scales),
        gu_bias=to_dev(layer.gate_up_bias),
        d_blocks=to_dev(layer.down.blocks), d_scales=to_dev(layer.down.scales),
        d_bias=to_dev(layer.down_bias),
    )


def nvfp4_layer_to_device(layer):
    dev = layer_to_device(layer)
    dev["gu_scale2"] = to_dev(layer.gate_up.scale2)
    dev["d_scale2"] = to_dev(layer.down.scale2)
    return dev


def run_nvfp4_forward(moe, dev, ids, w, layer, flags=None, workspace=None):
    import torch
    ids_d = ids if isinstance(ids, torch.Tensor) else to_dev(ids.astype(np.int32))
    w_d = w if isinstance(w, torch.Tensor) else to_dev(w.astype(np.float32))
    if flags is None:
        flags = moe.MOE_FLAG_WEIGHT_ON_INPUT if layer.weight_on_input else 0
    out = moe.moe_nvfp4_forward_ex(dev["x"], ids_d, w_d, dev["gu_blocks"], dev["gu_scales"],
                                   dev["gu_scale2"], dev["gu_bias"], dev["d_blocks"], dev["d_scales"],
                                   dev["d_scale2"], dev["d_bias"], alpha=layer.alpha, limit=layer.limit,
                                   flags=flags, workspace=workspace)
    torch.cuda.synchronize()
    return out


def oracle_nvfp4_forward(oracle, layer, ids, w, tokens=None, envelope=False):
    return oracle.nvfp4_forward_tokens(layer.x_bits, ids, w, layer.gate_up.blocks, layer.gate_up.scales,
                                       layer.gate_up.scale2, layer.gate_up_bias, layer.down.blocks,
                                       layer.down.scales, layer.down.scale2, layer.down_bias,
                                       alpha=layer.alpha, limit=layer.limit,
                                       weight_on_input=layer.weight_on_input, tokens=tokens,
                                       envelope=envelope)


def bf16_tensor_to_f64(t):
    import torch
    bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bits_of(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def run_forward(moe, dev, ids, w, layer, flags=None, workspace=None):
    import torch
    ids_d = ids if isinstance(ids, torch.Tensor) else to_dev(ids.astype(np.int32))
    w_d = w if isinstance(w, torch.Tensor) else to_dev(w.astype(np.float32))
    if flags is None:
        flags = moe.MOE_FLAG_WEIGHT_ON_INPUT if layer.weight_on_input else 0
    out = moe.moe_mxfp4_forward_ex(dev["x"], ids_d, w_d, dev["gu_blocks"], dev["gu_scales"],
                                   dev["gu_bias"], dev["d_blocks"], dev["d_scales"], dev["d_bias"],
                                   alpha=layer.alpha, limit=layer.limit, flags=flags,
                                   workspace=workspace)
    torch.cuda.synchronize()
    return out


def oracle_forward(oracle, layer, ids, w, tokens=None, envelope=False):
    return oracle.forward_tokens(layer.x_bits, ids, w, layer.gate_up.blocks, layer.gate_up.scales,
                                 layer.gate_up_bias, layer.down.blocks, layer.down.scales,
                                 layer.down_bias, alpha=layer.alpha, limit=layer.limit,
                                 weight_on_input=layer.weight_on_input, tokens=tokens,
                                 envelope=envelope)


def sample_tokens(T, n, seed=0):
    if T <= n:
        return np.arange(T, dtype=np.int64)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, T - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, T - 1], mid])).astype(np.int64)


def stratified_tokens(ids, E, tile_rows, extra=8, seed=0):
    """Tokens to compare at full size, chosen so that the sample reaches every tile the
    grouped kernels form: pairs p = t*k + j are grouped by expert in ascending p (the
    permutation's stable order), each expert's rows are cut into token tiles of
    `tile_rows`, and the tokens of the first and the last row of every tile of every
    touched expert are taken (so every touched expert, every full tile and every
    ragged tail), plus `extra` random tokens.  Bookkeeping only: no layer arithmetic."""
    ids = np.asarray(ids)
    T, k = ids.shape
    flat = ids.reshape(-1)
    picked = set()
    for e in range(E):
        pairs = np.nonzero(flat == e)[0]          # ascending p
        for r0 in range(0, pairs.size, tile_rows):
            r1 = min(r0 + tile_rows, pairs.size) - 1
            picked.add(int(pairs[r0]) // k)
            picked.add(int(pairs[r1]) // k)
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(T), np.fromiter(picked, dtype=np.int64, count=len(picked)))
    if rest.size and extra:
        picked.update(int(t) for t in rng.choice(rest, size=min(extra, rest.size), replace=False))
    return np.sort(np.fromiter(picked, dtype=np.int64, count=len(picked)))
