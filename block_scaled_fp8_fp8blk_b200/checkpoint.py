"""Serialized block-FP8 checkpoints: what the converter writes and the loader reads.

FastVideo PR #1829 ("MiniMax H3: block-FP8 text encoder on Hopper, its
converter, and a 4xH100 FastH3 profile"), section "Changes", converter
bullet: the checkpoint holds each linear's E4M3 weight plus its
[N/128, K/128] ``weight_scale_inv``, a ``quantization_config`` in
``config.json`` and a regenerated index. The page gives no schema; this
module takes the plainest reading of those words:

* tensors in safetensors files (an 8-byte little-endian header length, a JSON
  header naming each tensor's dtype, shape and byte range, then the raw
  little-endian bytes), sharded as ``model-XXXXX-of-YYYYY.safetensors``;
* a linear ``<p>.weight`` becomes ``<p>.weight`` (dtype ``F8_E4M3``, shape
  [N, K], codes unpadded) and ``<p>.weight_scale_inv`` (``F32``,
  [ceil(N/128), ceil(K/128)]); every other tensor is kept as it is;
* ``model.safetensors.index.json`` maps every tensor to its shard and states
  the total byte size;
* ``config.json`` gains ``quantization_config`` = :data:`QUANTIZATION_CONFIG`
  (E4M3 weights in 128 x 128 blocks, activations quantized at run time).

Host-side I/O only; the conversion itself runs in ``fp8blk_quantize_weight``
on the GPU (there is no CPU path: :func:`quantize_state_dict` raises without
one).
"""
from __future__ import annotations

import json
import os
import struct
from typing import Callable, Iterable

import torch

__all__ = [
    "QUANTIZATION_CONFIG", "INDEX_NAME", "write_safetensors", "read_safetensors",
    "default_is_linear", "quantize_state_dict", "save_checkpoint", "load_checkpoint",
    "convert_checkpoint", "linear_weights",
]

QUANTIZATION_CONFIG = {
    "quant_method": "fp8",
    "fmt": "e4m3",
    "weight_block_size": [128, 128],
    "activation_scheme": "dynamic",
}
INDEX_NAME = "model.safetensors.index.json"
SCALE_SUFFIX = "_scale_inv"

# safetensors dtype names <-> torch dtypes
_DTYPES = {
    "F8_E4M3": torch.float8_e4m3fn, "F32": torch.float32, "F16": torch.float16,
    "BF16": torch.bfloat16, "F64": torch.float64, "U8": torch.uint8, "I8": torch.int8,
    "I16": torch.int16, "I32": torch.int32, "I64": torch.int64, "BOOL": torch.bool,
}
_NAMES = {v: k for k, v in _DTYPES.items()}


def write_safetensors(path: str, tensors: dict, metadata: dict | None = None) -> int:
    """Writes ``tensors`` (name -> tensor, any device) to one safetensors
    file; returns the bytes of tensor data written. Tensors are stored in
    name order, contiguous, after a JSON header padded with spaces to a
    multiple of 8 bytes."""
    header, blobs, off = {}, [], 0
    if metadata:
        header["__metadata__"] = {str(k): str(v) for k, v in metadata.items()}
    for name in sorted(tensors):
        t = tensors[name].detach().contiguous().cpu()
        if t.dtype not in _NAMES:
            raise ValueError(f"{name}: dtype {t.dtype} has no safetensors name")
        raw = t.reshape(-1).view(torch.uint8).numpy().tobytes() if t.numel() else b""
        header[name] = {"dtype": _NAMES[t.dtype], "shape": list(t.shape),
                        "data_offsets": [off, off + len(raw)]}
        blobs.append(raw)
        off += len(raw)
    h = json.dumps(header, separators=(",", ":")).encode()
    h += b" " * (-len(h) % 8)
    tmp = path + ".tmp"
    with open(tmp, "wb") as f:
        f.write(struct.pack("<Q", len(h)))
        f.write(h)
        for b in blobs:
            f.write(b)
    os.replace(tmp, path)
    return off


def read_safetensors(path: str, names: Iterable[str] | None = None) -> dict:
    """Reads tensors (all, or ``names``) of one safetensors file into CPU tensors."""
    with open(path, "rb") as f:
        (n,) = struct.unpack("<Q", f.read(8))
        header = json.loads(f.read(n))
        base = 8 + n
        want = [k for k in header if k != "__metadata__"] if names is None else list(names)
        out = {}
        for name in want:
            rec = header[name]
            dt = _DTYPES[rec["dtype"]]
            b0, b1 = rec["data_offsets"]
            f.seek(base + b0)
            raw = bytearray(f.read(b1 - b0))
            if len(raw) != b1 - b0:
                raise ValueError(f"{path}: {name} is truncated")
            t = torch.frombuffer(raw, dtype=torch.uint8) if raw else torch.empty(0, dtype=torch.uint8)
            out[name] = t.view(dt).reshape(rec["shape"])
    return out


def default_is_linear(name: str, t: torch.Tensor) -> bool:
    """The converter's default choice of the weights it quantizes: 2-D
    ``*.weight`` tensors other than embeddings, norms and the LM head (the
    page quantizes the language model's linears)."""
    if t.dim() != 2 or not name.endswith(".weight"):
        return False
    return not any(k in name for k in ("embed", "norm", "lm_head"))


def quantize_state_dict(state: dict, is_linear: Callable = default_is_linear,
                        device: str | torch.device = "cuda") -> dict:
    """Converts every linear weight of ``state`` with the GPU converter
    (``fp8blk_quantize_weight``): ``<p>.weight`` -> E4M3 codes [N, K] (dtype
    float8_e4m3fn, CPU) + ``<p>.weight_scale_inv`` float32; other tensors are
    returned unchanged. Raises without a CUDA device when there is a linear
    to convert (there is no CPU path)."""
    import block_scaled_fp8_fp8blk_b200 as fb
    out = {}
    for name, t in state.items():
        if not is_linear(name, t):
            out[name] = t
            continue
        if not torch.cuda.is_available():
            raise RuntimeError("quantize_state_dict needs a CUDA device (the converter is a GPU kernel)")
        w = t.detach().to(device=device, dtype=torch.bfloat16).contiguous()
        N, K = w.shape
        ldw = -(-K // 8) * 8
        if ldw != K:  # the converter wants a 16-byte row pitch
            wp = torch.zeros((N, ldw), dtype=torch.bfloat16, device=device)
            wp[:, :K] = w
            w = wp[:, :K]
        q, s = fb.quantize_weight(w)
        out[name] = q.contiguous().cpu().view(torch.float8_e4m3fn)
        out[name + SCALE_SUFFIX] = s.cpu()
    return out


def save_checkpoint(out_dir: str, tensors: dict, config: dict | None = None,
                    max_shard_bytes: int = 5 * 10**9) -> dict:
    """Writes ``tensors`` as safetensors shards (name order, each shard up to
    ``max_shard_bytes`` unless one tensor is bigger), the index, and
    ``config.json`` with ``quantization_config`` when any tensor is E4M3.
    Returns the index."""
    os.makedirs(out_dir, exist_ok=True)
    groups, cur, cur_bytes = [], [], 0
    for name in sorted(tensors):
        nb = tensors[name].numel() * tensors[name].element_size()
        if cur and cur_bytes + nb > max_shard_bytes:
            groups.append(cur)
            cur, cur_bytes = [], 0
        cur.append(name)
        cur_bytes += nb
    if cur or not groups:
        groups.append(cur)
    weight_map, total = {}, 0
    for i, names in enumerate(groups):
        fname = f"model-{i + 1:05d}-of-{len(groups):05d}.safetensors"
        total += write_safetensors(os.path.join(out_dir, fname), {n: tensors[n] for n in names},
                                   metadata={"format": "pt"})
        for n in names:
            weight_map[n] = fname
    return _write_index_and_config(out_dir, weight_map, total, config,
                                   any(t.dtype == torch.float8_e4m3fn for t in tensors.values()))


def _write_index_and_config(out_dir: str, weight_map: dict, total: int, config: dict | None,
                            has_fp8: bool) -> dict:
    """The index (tensor -> shard, total bytes) and config.json, with
    quantization_config when the checkpoint holds E4M3 weights."""
    index = {"metadata": {"total_size": total}, "weight_map": dict(sorted(weight_map.items()))}
    with open(os.path.join(out_dir, INDEX_NAME), "w") as f:
        json.dump(index, f, indent=2)
    cfg = dict(config or {})
    if has_fp8:
        cfg["quantization_config"] = dict(QUANTIZATION_CONFIG)
    with open(os.path.join(out_dir, "config.json"), "w") as f:
        json.dump(cfg, f, indent=2)
    return index


def _read_config(directory: str) -> dict:
    """config.json of a checkpoint directory, or {} when it has none."""
    path = os.path.join(directory, "config.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        return json.load(f)


def load_checkpoint(in_dir: str, names: Iterable[str] | None = None) -> tuple[dict, dict]:
    """Reads a checkpoint written by :func:`save_checkpoint` (or any
    directory with the same index): returns (CPU tensors, config)."""
    with open(os.path.join(in_dir, INDEX_NAME)) as f:
        index = json.load(f)
    wm = index["weight_map"]
    want = list(wm) if names is None else list(names)
    by_file: dict = {}
    for n in want:
        by_file.setdefault(wm[n], []).append(n)
    out = {}
    for fname, ns in by_file.items():
        out.update(read_safetensors(os.path.join(in_dir, fname), ns))
    return out, _read_config(in_dir)


def convert_checkpoint(src_dir: str, dst_dir: str, is_linear: Callable = default_is_linear,
                       max_shard_bytes: int = 5 * 10**9) -> dict:
    """BF16 checkpoint (index + shards, or a single ``model.safetensors``) ->
    block-FP8 checkpoint. Source shards are converted one at a time on the
    GPU and output shards are written as they fill, so the host holds at most
    one source shard, its converted tensors and one output shard (each output
    shard up to ``max_shard_bytes`` unless one tensor is bigger). Shards are
    written under temporary names and renamed model-XXXXX-of-YYYYY once their
    count is known; returns the index."""
    idx_path = os.path.join(src_dir, INDEX_NAME)
    if os.path.exists(idx_path):
        with open(idx_path) as f:
            files = sorted(set(json.load(f)["weight_map"].values()))
    else:
        files = ["model.safetensors"]
    os.makedirs(dst_dir, exist_ok=True)
    parts: list = []          # (temporary file name, tensor names)
    pending: dict = {}
    state = {"bytes": 0, "total": 0, "fp8": False}

    def write_part():
        tmp = f"model-part-{len(parts):05d}.safetensors"
        state["total"] += write_safetensors(os.path.join(dst_dir, tmp), pending,
                                            metadata={"format": "pt"})
        parts.append((tmp, sorted(pending)))
        pending.clear()
        state["bytes"] = 0

    for fname in files:
        converted = quantize_state_dict(read_safetensors(os.path.join(src_dir, fname)), is_linear)
        for name in sorted(converted):
            t = converted[name]
            nb = t.numel() * t.element_size()
            if pending and state["bytes"] + nb > max_shard_bytes:
                write_part()
            pending[name] = t
            state["bytes"] += nb
            state["fp8"] = state["fp8"] or t.dtype == torch.float8_e4m3fn
        del converted
    if pending or not parts:
        write_part()
    weight_map = {}
    for i, (tmp, names) in enumerate(parts):
        final = f"model-{i + 1:05d}-of-{len(parts):05d}.safetensors"
        os.replace(os.path.join(dst_dir, tmp), os.path.join(dst_dir, final))
        for n in names:
            weight_map[n] = final
    return _write_index_and_config(dst_dir, weight_map, state["total"], _read_config(src_dir),
                                   state["fp8"])


def linear_weights(tensors: dict, name: str, device: str | torch.device = "cuda",
                   pin: bool = False):
    """(q, scale_inv) of linear ``name`` laid out for the fp8blk calls: q a
    uint8 [N, K] view of an [N, ldq] buffer with ldq = K rounded up to 16
    (on ``device``, or pinned host memory with ``pin`` for
    fp8blk_streamed_linears), scale_inv float32 [ceil(N/128), ceil(K/128)]."""
    q = tensors[name].view(torch.uint8)
    s = tensors[name + SCALE_SUFFIX].to(torch.float32)
    N, K = q.shape
    ldq = -(-K // 16) * 16
    if pin:
        buf = torch.zeros((N, ldq), dtype=torch.uint8, pin_memory=True)
        buf[:, :K] = q
        return buf[:, :K], s.contiguous().pin_memory()
    buf = torch.zeros((N, ldq), dtype=torch.uint8, device=device)
    buf[:, :K] = q.to(device)
    return buf[:, :K], s.to(device).contiguous()
