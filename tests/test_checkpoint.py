"""Checkpoint I/O of the converter (host side, no GPU): the safetensors files
are checked against the independent `safetensors` package in both
directions, and the sharded save / load, the index and the
quantization_config are checked for a round trip."""
import json
import os
import struct

import pytest
import torch
import safetensors.torch as st

from block_scaled_fp8_fp8blk_b200 import checkpoint as ck


def sample_tensors(seed=0):
    g = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 256, (300, 1000), generator=g, dtype=torch.uint8)
    codes[codes & 0x7F == 0x7F] = 0x12                       # no NaN codes
    return {
        "model.layers.0.mlp.down_proj.weight": codes.view(torch.float8_e4m3fn),
        "model.layers.0.mlp.down_proj.weight_scale_inv": torch.rand(3, 8, generator=g),
        "model.embed_tokens.weight": torch.randn(50, 64, generator=g).to(torch.bfloat16),
        "model.norm.weight": torch.randn(64, generator=g).to(torch.bfloat16),
        "model.rope.inv_freq": torch.rand(32, generator=g, dtype=torch.float64),
        "model.steps": torch.tensor([3, 1, 4], dtype=torch.int64),
        "model.mask": torch.tensor([True, False, True]),
        "model.empty": torch.empty(0, 5),
    }


def same(a, b):
    assert a.dtype == b.dtype and a.shape == b.shape
    assert torch.equal(a.reshape(-1).view(torch.uint8), b.reshape(-1).view(torch.uint8))


def test_written_file_reads_with_safetensors(tmp_path):
    t = sample_tensors()
    p = str(tmp_path / "a.safetensors")
    ck.write_safetensors(p, t, metadata={"format": "pt"})
    back = st.load_file(p)
    assert set(back) == set(t)
    for k in t:
        same(back[k], t[k])


def test_reads_file_written_by_safetensors(tmp_path):
    t = sample_tensors(1)
    p = str(tmp_path / "b.safetensors")
    st.save_file(t, p)
    back = ck.read_safetensors(p)
    assert set(back) == set(t)
    for k in t:
        same(back[k], t[k])
    part = ck.read_safetensors(p, ["model.norm.weight"])
    assert list(part) == ["model.norm.weight"]


def test_header_layout(tmp_path):
    t = sample_tensors(2)
    p = str(tmp_path / "c.safetensors")
    total = ck.write_safetensors(p, t)
    raw = open(p, "rb").read()
    (n,) = struct.unpack("<Q", raw[:8])
    assert n % 8 == 0
    header = json.loads(raw[8:8 + n])
    spans = sorted(v["data_offsets"] for k, v in header.items() if k != "__metadata__")
    assert spans[0][0] == 0 and spans[-1][1] == total == len(raw) - 8 - n
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0                                         # contiguous, no gaps
    assert header["model.layers.0.mlp.down_proj.weight"]["dtype"] == "F8_E4M3"
    assert header["model.layers.0.mlp.down_proj.weight_scale_inv"]["shape"] == [3, 8]


def test_sharded_round_trip_index_and_config(tmp_path):
    t = sample_tensors(3)
    out = str(tmp_path / "ckpt")
    index = ck.save_checkpoint(out, t, config={"hidden_size": 64}, max_shard_bytes=200_000)
    files = sorted(set(index["weight_map"].values()))
    assert len(files) >= 2
    assert all(f.endswith(f"-of-{len(files):05d}.safetensors") for f in files)
    assert set(index["weight_map"]) == set(t)
    assert index["metadata"]["total_size"] == sum(v.numel() * v.element_size() for v in t.values())
    on_disk = json.load(open(os.path.join(out, ck.INDEX_NAME)))
    assert on_disk == index
    back, cfg = ck.load_checkpoint(out)
    for k in t:
        same(back[k], t[k])
    assert cfg["hidden_size"] == 64
    assert cfg["quantization_config"] == {"quant_method": "fp8", "fmt": "e4m3",
                                          "weight_block_size": [128, 128],
                                          "activation_scheme": "dynamic"}
    # every shard also reads with the safetensors package
    for f in files:
        for k, v in st.load_file(os.path.join(out, f)).items():
            same(v, t[k])


def test_no_quantization_config_without_fp8(tmp_path):
    out = str(tmp_path / "bf16")
    ck.save_checkpoint(out, {"a.weight": torch.ones(4, 4, dtype=torch.bfloat16)})
    assert "quantization_config" not in json.load(open(os.path.join(out, "config.json")))


def test_linear_weights_pitch():
    t = sample_tensors(4)
    q, s = ck.linear_weights(t, "model.layers.0.mlp.down_proj.weight", device="cpu")
    assert q.shape == (300, 1000) and q.stride(0) == 1008 and q.dtype == torch.uint8
    assert torch.equal(q, t["model.layers.0.mlp.down_proj.weight"].view(torch.uint8))
    assert torch.equal(s, t["model.layers.0.mlp.down_proj.weight_scale_inv"])


def test_default_linear_choice():
    f = ck.default_is_linear
    assert f("model.layers.3.self_attn.q_proj.weight", torch.empty(8, 8))
    assert f("model.layers.3.mlp.gate_up_proj.weight", torch.empty(8, 8))
    assert not f("model.embed_tokens.weight", torch.empty(8, 8))
    assert not f("model.layers.3.input_layernorm.weight", torch.empty(8))
    assert not f("lm_head.weight", torch.empty(8, 8))
    assert not f("model.layers.3.self_attn.q_proj.bias", torch.empty(8, 8))


def test_quantize_state_dict_needs_a_gpu(monkeypatch):
    monkeypatch.setattr(torch.cuda, "is_available", lambda: False)
    with pytest.raises(RuntimeError, match="CUDA"):
        ck.quantize_state_dict({"l.weight": torch.ones(4, 4)})


def test_convert_checkpoint_without_linears_passes_through(tmp_path, monkeypatch):
    """With nothing to quantize no GPU is needed: the converter re-shards the
    tensors unchanged and keeps the source config (no quantization_config,
    since no tensor is E4M3)."""
    monkeypatch.setattr(torch.cuda, "is_available", lambda: False)
    g = torch.Generator().manual_seed(9)
    src_t = {"model.norm.weight": torch.randn(64, generator=g).to(torch.bfloat16),
             "model.embed_tokens.weight": torch.randn(40, 16, generator=g).to(torch.bfloat16),
             "model.layers.0.mlp.up_proj.weight": torch.randn(8, 8, generator=g).to(torch.bfloat16)}
    src = str(tmp_path / "src")
    ck.save_checkpoint(src, src_t, {"model_type": "toy", "hidden_size": 16}, max_shard_bytes=200)
    dst = str(tmp_path / "dst")
    idx = ck.convert_checkpoint(src, dst, is_linear=lambda n, t: False, max_shard_bytes=10**6)
    assert set(idx["weight_map"]) == set(src_t)
    assert len(set(idx["weight_map"].values())) == 1          # one shard at the larger limit
    back, cfg = ck.load_checkpoint(dst)
    assert cfg == {"model_type": "toy", "hidden_size": 16}
    for k, v in src_t.items():
        same(back[k], v)
    with pytest.raises(RuntimeError, match="CUDA"):           # a linear still needs the GPU
        ck.convert_checkpoint(src, str(tmp_path / "dst2"))


def test_convert_checkpoint_writes_shards_as_they_fill(tmp_path, monkeypatch):
    """Output shards are written while converting, each up to the size limit
    (one tensor larger than the limit gets a shard of its own), renamed
    model-XXXXX-of-YYYYY at the end with no temporary file left behind; the
    index covers every tensor once."""
    monkeypatch.setattr(torch.cuda, "is_available", lambda: False)
    g = torch.Generator().manual_seed(10)
    src_t = {f"model.layers.{i}.norm.weight": torch.randn(16 * (i + 1), generator=g).to(torch.bfloat16)
             for i in range(7)}
    src_t["model.embed_tokens.weight"] = torch.randn(30, 20, generator=g).to(torch.bfloat16)  # 1200 B
    src = str(tmp_path / "src")
    ck.save_checkpoint(src, src_t, {"model_type": "toy"}, max_shard_bytes=100)
    dst = str(tmp_path / "dst")
    limit = 300
    idx = ck.convert_checkpoint(src, dst, is_linear=lambda n, t: False, max_shard_bytes=limit)
    files = sorted(set(idx["weight_map"].values()))
    assert len(files) >= 3
    assert files == [f"model-{i + 1:05d}-of-{len(files):05d}.safetensors" for i in range(len(files))]
    assert sorted(os.listdir(dst)) == sorted(files + [ck.INDEX_NAME, "config.json"])
    assert set(idx["weight_map"]) == set(src_t)
    for f in files:
        names = [n for n, v in idx["weight_map"].items() if v == f]
        nbytes = sum(src_t[n].numel() * 2 for n in names)
        assert nbytes <= limit or len(names) == 1
    assert idx["metadata"]["total_size"] == sum(t.numel() * 2 for t in src_t.values())
    back, _ = ck.load_checkpoint(dst)
    for k, v in src_t.items():
        same(back[k], v)
