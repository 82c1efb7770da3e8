"""Host-side helpers of bench.py (no GPU): the fingerprint that keys the
recorded DRAM traffic of a decode call to the code that call runs."""
import json
import os

import bench


def test_every_named_definition_is_found():
    for split in (False, True):
        for cascade in (False, True):
            fp = bench.decode_code_sha(split, cascade)
            assert len(fp) == 16 and int(fp, 16) >= 0


def test_definitions_skip_calls_and_declarations():
    src = ("int f(int a);\n"
           "int g() { return f(1); }\n"
           "template <int N>\n"
           "__device__ int f(int a)\n"
           "{\n"
           "    if (a) { return a; }\n"
           "    return N;\n"
           "}\n"
           "struct S { int x; };\n")
    (fdef,) = bench._definitions(src, "f")
    assert fdef.startswith("template <int N>") and fdef.endswith("return N;\n}")
    (sdef,) = bench._definitions(src, "S")
    assert sdef == "struct S { int x; }"


def test_fingerprint_depends_on_the_code_it_covers(tmp_path):
    root = tmp_path
    csrc = root / bench.CSRC
    csrc.mkdir(parents=True)
    for name in ("pkv_ptx.cuh", "pkv_kernels.cuh", "pkv_prefill.cuh", "pagedkv.cu"):
        (csrc / name).write_text(open(os.path.join(bench.ROOT, bench.CSRC, name)).read())
    same = bench.decode_code_sha(False, False, root=str(root))
    assert same == bench.decode_code_sha(False, False)
    # an edit inside the decode kernel changes it; one in the copy kernel does not
    k = (csrc / "pkv_kernels.cuh").read_text()
    edited = k.replace("copy_blocks_kernel(", "copy_blocks_kernel(/* x */", 1)
    (csrc / "pkv_kernels.cuh").write_text(edited)
    assert bench.decode_code_sha(False, False, root=str(root)) == same
    edited = edited.replace("paged_decode_kernel(", "paged_decode_kernel(/* x */", 1)
    (csrc / "pkv_kernels.cuh").write_text(edited)
    assert bench.decode_code_sha(False, False, root=str(root)) != same


def test_committed_traffic_entries_are_well_formed():
    with open(bench.TRAFFIC_FILE) as f:
        d = json.load(f)
    for name, entry in d.items():
        if name == "note":
            continue
        assert entry["dram_bytes_per_launch"] > 0 and len(entry["source_sha"]) == 16


def test_packed_inputs_round_trip_at_aligned_offsets():
    """The end-to-end step uploads its inputs as one packed buffer: every
    tensor sits at a 256-byte aligned offset and reads back unchanged through
    its view, after a byte copy of the whole buffer."""
    import torch
    src = {"query": torch.randn(3, 4, 8).to(torch.bfloat16),
           "slot_mapping": torch.arange(5, dtype=torch.int64) * 7,
           "block_tables": torch.arange(12, dtype=torch.int32).view(3, 4),
           "context_lens": torch.tensor([1, 2, 3], dtype=torch.int32)}
    hbuf, hview = bench._packed(src, lambda n: torch.zeros(n, dtype=torch.uint8))
    for k, v in src.items():
        hview[k].copy_(v)
    dbuf, dview = bench._packed(src, lambda n: torch.full((n,), 255, dtype=torch.uint8))
    dbuf.copy_(hbuf)
    for k, v in src.items():
        assert dview[k].shape == v.shape and dview[k].dtype == v.dtype
        assert (dview[k].storage_offset() * dview[k].element_size()) % 256 == 0
        assert torch.equal(dview[k], v), k
    assert hbuf.numel() % 256 == 0
