"""The benchmark's per-workload oracle timings (bench.cpu_baseline_secondary) on small CPU
inputs: each kind returns a positive rate in its unit and an extrapolated full-workload time,
and a failure is reported in the entry instead of raised."""
import dataclasses
import importlib.util
import os
import types

import pytest
import torch

from global_attention_sink_softmax_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def runner(w, d, bytes_, flops, workload):
    return types.SimpleNamespace(w=w, d=d, bytes=bytes_, flops=flops, workload=workload)


def check(e, unit):
    assert "error" not in e, e
    assert e["unit"] == unit and e["value"] > 0 and e["kind"] == "oracle"
    assert e["full_workload_s_extrapolated"] > 0 and e["cores"] >= 1


def test_prefill_and_chunk(bench):
    w = dataclasses.replace(W.GA_PREFILL, L=300)
    d = W.prefill_inputs(w)
    fl, by = bench.prefill_counts(w)
    check(bench.cpu_baseline_secondary("prefill", runner(w, d, by, fl, w.name), 0.2), "TFLOP/s")
    wc = dataclasses.replace(W.GA_CHUNK, L=100, prefix=200)
    dc = W.prefill_inputs(wc, L=300)
    dc["q"] = dc["q"][:, 200:]
    fl, by = bench.prefill_counts(wc)
    check(bench.cpu_baseline_secondary("prefill", runner(wc, dc, by, fl, wc.name), 0.2), "TFLOP/s")


def test_rope(bench):
    w = dataclasses.replace(W.SWA_PREFILL, B=1, L=64)
    d = W.prefill_inputs(w)
    e = bench.cpu_baseline_secondary("rope", runner(w, d, 10 ** 9, 10 ** 9, "rope"), 0.2)
    check(e, "GB/s")
    assert e["cores"] == 1


@pytest.mark.parametrize("fp8", [False, True])
def test_decode(bench, fp8):
    w = dataclasses.replace(W.GA_DECODE, B=3, ctx=200)
    d = W.decode_inputs(w, fp8=fp8)
    fl, by = bench.decode_counts(w, d)
    check(bench.cpu_baseline_secondary("decode", runner(w, d, by, fl, w.name)), "GB/s")
    wr = dataclasses.replace(W.SWA_DECODE, B=20)
    dr = W.decode_inputs(wr)
    fl, by = bench.decode_counts(wr, dr)
    check(bench.cpu_baseline_secondary("decode", runner(wr, dr, by, fl, wr.name)), "GB/s")


def test_failure_is_reported_not_raised(bench):
    w = dataclasses.replace(W.GA_DECODE, B=2, ctx=10)
    e = bench.cpu_baseline_secondary("decode", runner(w, {}, 1, 1, "broken"))
    assert e["kind"] == "oracle" and "error" in e


def test_headline_baseline_reports_its_extrapolation(bench):
    w = dataclasses.replace(W.SWA_PREFILL, B=1, L=512)
    d = W.prefill_inputs(w)
    e = bench.cpu_baseline_prefill(w, d, target_s=0.2)
    assert e["unit"] == "TFLOP/s" and e["value"] > 0 and e["kind"] == "oracle"
    assert e["full_workload_s_extrapolated"] > 0
