"""Host logic of bench.py that needs no GPU: the DRAM-traffic figure of the BERT line.

One ncu capture of the three attention kernels at the BERT-base layer-0 shape (32 sequences x 12
heads x 512 keys: 94,906,368 bytes) is scaled to a whole cascade step by the step's kept keys x
kept heads.  The keep schedule (k_l = ceil(512 * 0.9^l), heads 12, 12, 11, 11, 11, 10, 10, 10, 9,
9, 9, 8) gives 38,940 key-head units per sequence against the layer-0 shape's 6,144, so the step
figure is 94,906,368 * 38,940 / 6,144 = 601,506,180 bytes.  The figure is null once the kernel
sources differ from those the capture was taken on, or when they cannot be read."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from cascade_token_head_b200 import synth  # noqa: E402


def test_bert_step_traffic_scaling(monkeypatch):
    captured = bench.CAPTURED_TRAFFIC["prefill_attention_layer"]
    assert captured["bytes"] == 94_906_368 and captured["kept_key_heads"] == 512 * 12
    w = synth.bert_base_prefill()
    assert sum(k * h for k, h in zip(w.token_keep, w.head_keep)) == 38_940
    monkeypatch.setattr(bench, "sources_hash", lambda *a, **k: captured["sources_sha256"])
    t, why = bench.prefill_traffic(w)
    assert t == pytest.approx(601_506_180, rel=0, abs=1e-3)
    assert "scaled" in why


def test_traffic_null_without_capture_or_after_a_change(monkeypatch):
    captured = bench.CAPTURED_TRAFFIC["prefill_attention_layer"]
    monkeypatch.setattr(bench, "sources_hash", lambda *a, **k: captured["sources_sha256"])
    t, why = bench.prefill_traffic(synth.long_prefill())
    assert t is None and "no DRAM capture" in why
    monkeypatch.setattr(bench, "sources_hash", lambda *a, **k: "0" * 16)
    t, why = bench.prefill_traffic(synth.bert_base_prefill())
    assert t is None and "changed" in why

    def unreadable(*a, **k):
        raise OSError("no sources")

    monkeypatch.setattr(bench, "sources_hash", unreadable)
    t, why = bench.prefill_traffic(synth.bert_base_prefill())
    assert t is None and "not beside" in why
