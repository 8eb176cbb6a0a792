"""Host checks of the bench's algorithmic byte counts, the numerators of every
roofline fraction it reports.  The expected figures are worked out by hand
from the workload shapes, not from the counting code:

  encoder, fp32, fused step, per query (Lq = S: one query per pixel):
    offsets and logits   8 heads x 16 samples x (8 + 4) B     = 1536
    output               8 heads x 32 channels x 4 B          = 1024
    reference point      2 x 4 B                              =    8
    value, read once     8 heads x 32 channels x 4 B / pixel  = 1024
                                                               = 3592 B
  encoder, bf16 value: the value term halves                  = 3080 B
  stress (K = 8, bf16): 8 x 32 x 12 + 1024 + 8 + 512           = 4616 B
The split step's forward also writes the locations and weights (12 B per
sample, +1536 B per encoder query).  The backward reads value, locations,
weights and grad_out and writes grad_value, grad locations and grad weights:
for the encoder 36.5 + 54.7 + 36.5 + 36.5 + 54.7 MB = 219.0 MB."""
import bench
from scale_deformable_attention_02_b200 import workloads as wl


def test_fused_forward_bytes_per_query():
    for w, per_query in ((wl.ENCODER, 3592), (wl.ENCODER_BF16, 3080), (wl.STRESS, 4616)):
        ab = bench.algorithmic_bytes(w, "fused")
        assert ab["fwd"] == per_query * w.N * w.queries, (w.name, ab["fwd"])


def test_split_forward_adds_the_saved_locations_and_weights():
    w = wl.ENCODER
    samples = w.N * w.queries * w.M * w.L * w.K
    assert (bench.algorithmic_bytes(w, "split")["fwd"]
            == bench.algorithmic_bytes(w, "fused")["fwd"] + 12 * samples)


def test_backward_bytes():
    enc = bench.algorithmic_bytes(wl.ENCODER, "split")["bwd"]
    assert enc == 218_984_448  # 219.0 MB, as worked out above
    stress = bench.algorithmic_bytes(wl.STRESS, "split")["bwd"]
    # bf16 value 152 MB + locations and weights 913 MB + grad_out 304 MB
    # + grad_value 304 MB + grad locations and weights 913 MB
    assert abs(stress - 2.587e9) < 1e6


def test_touched_rows_replace_the_full_map():
    """With the count of value rows some sample touches, the value term is
    those rows once (the decoder reads only part of the map)."""
    w = wl.DECODER
    full = bench.algorithmic_bytes(w, "split")
    part = bench.algorithmic_bytes(w, "split", touched_rows=1000)
    rows = w.N * w.S * w.M
    assert full["fwd"] - part["fwd"] == (rows - 1000) * w.D * 4


def test_kernel_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    """The recorded DRAM traffic is keyed by a hash of the kernels' device
    code: a comment edit keeps it, a code edit changes it."""
    import os
    import shutil
    src = os.path.join(bench.ROOT, "scale_deformable_attention_02_b200", "csrc")
    dst = tmp_path / "scale_deformable_attention_02_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_hash()
    f = dst / "msda_bwd.cu"
    text = f.read_text()
    f.write_text(text.replace("namespace msda {", "// a remark\nnamespace msda { /* another */", 1))
    assert bench.kernel_source_hash() == base
    f.write_text(text.replace("constexpr int kWarps = 8;", "constexpr int kWarps = 4;", 1))
    assert bench.kernel_source_hash() != base


def test_traffic_entries_cover_the_default_configurations():
    """The default line (split step, untiled calls) and the fused step look up
    entries that profiles/traffic.json holds, and the tiled schedule never
    reads the untiled kernels' counts."""
    import json
    import os
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)
    assert bench.traffic_key("encoder", "split", "untiled") == "encoder"
    assert bench.traffic_key("encoder", "fused", "untiled") == "encoder/fused"
    assert bench.traffic_key("encoder", "split", "tiled") == "encoder/tiled"
    for key in ("encoder", "encoder/fused"):
        assert {"fwd", "bwd"} <= set(entries[key]), key
    assert "encoder/tiled" not in entries


def test_untiled_hash_ignores_the_tiled_sources(tmp_path, monkeypatch):
    """Counters of the untiled kernels stay valid when only the tiled kernels
    change, and the tiled schedule's hash tracks both."""
    import os
    import shutil
    src = os.path.join(bench.ROOT, "scale_deformable_attention_02_b200", "csrc")
    dst = tmp_path / "scale_deformable_attention_02_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    untiled, tiled = bench.kernel_source_hash(), bench.kernel_source_hash("tiled")
    f = dst / "msda_fwd_tiled.cu"
    f.write_text(f.read_text().replace("namespace msda {", "namespace msda { int unused_x;", 1))
    assert bench.kernel_source_hash() == untiled
    assert bench.kernel_source_hash("tiled") != tiled
