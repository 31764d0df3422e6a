"""Host logic of bench.py that the judged JSON line depends on (no GPU): the
traffic field is taken from the committed ncu summary only while the kernel
sources still hash to the captured revision and the dispatched kernel is the
captured one."""
import os
import shutil

import bench


def _summary(tmp_path, kernel, sha, traffic="123456"):
    p = tmp_path / "summary.md"
    p.write_text("# a kernel\n\nsome text: with a colon\n\n"
                 f"- kernel: `{kernel}`\n"
                 f"- traffic_bytes_per_launch: `{traffic}`\n"
                 f"- source_sha256: `{sha}`\n")
    return str(p)


def test_traffic_read_when_sources_and_kernel_match(tmp_path):
    path = _summary(tmp_path, "prefill_seq_kernel", bench.kernel_source_sha256())
    assert bench.captured_traffic("prefill_seq_kernel", path) == 123456


def test_traffic_null_after_a_kernel_change(tmp_path):
    path = _summary(tmp_path, "prefill_seq_kernel", "0" * 64)
    assert bench.captured_traffic("prefill_seq_kernel", path) is None


def test_traffic_null_for_another_kernel(tmp_path):
    path = _summary(tmp_path, "prefill_tc_kernel<128>", bench.kernel_source_sha256())
    assert bench.captured_traffic("prefill_seq_kernel", path) is None


def test_traffic_null_when_summary_missing_or_malformed(tmp_path):
    assert bench.captured_traffic("prefill_seq_kernel", str(tmp_path / "absent.md")) is None
    path = _summary(tmp_path, "prefill_seq_kernel", bench.kernel_source_sha256(), traffic="n/a")
    assert bench.captured_traffic("prefill_seq_kernel", path) is None


def test_source_hash_covers_kernel_code_only(tmp_path, monkeypatch):
    # a copy of the source tree: host code (lightning.cu) and comments in the
    # kernel headers may change without invalidating a capture, kernel code
    # may not
    src = os.path.join(bench.ROOT, "linear_attention_13_b200", "csrc")
    dst = tmp_path / "linear_attention_13_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha256()
    assert len(h0) == 64
    (dst / "lightning.cu").write_text((dst / "lightning.cu").read_text() + "\nstatic int host_edit = 1;\n")
    assert bench.kernel_source_sha256() == h0
    text = (dst / "decode.cuh").read_text()
    (dst / "decode.cuh").write_text(text + "\n// a comment\n/* and a\n   block comment */\n")
    assert bench.kernel_source_sha256() == h0
    (dst / "decode.cuh").write_text(text + "\nstatic constexpr int kEdit = 1;\n")
    assert bench.kernel_source_sha256() != h0


def test_summary_source_files_limit_the_hash(tmp_path, monkeypatch):
    # a summary that names its kernel's headers stays valid when another
    # kernel's header changes, and not when one of its own does
    src = os.path.join(bench.ROOT, "linear_attention_13_b200", "csrc")
    dst = tmp_path / "linear_attention_13_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    files = {"common.cuh", "decode.cuh", "ptx.cuh"}
    path = tmp_path / "s.md"
    path.write_text("- kernel: `decode_step_kernel`\n- traffic_bytes_per_launch: `123`\n"
                    "- source_files: `common.cuh decode.cuh ptx.cuh`\n"
                    "- source_sha256: `%s`\n" % bench.kernel_source_sha256(files))
    assert bench.captured_traffic("decode_step_kernel", str(path)) == 123
    text = (dst / "prefill_tc.cuh").read_text()
    (dst / "prefill_tc.cuh").write_text(text + "\nstatic constexpr int kEdit = 1;\n")
    assert bench.captured_traffic("decode_step_kernel", str(path)) == 123
    text = (dst / "decode.cuh").read_text()
    (dst / "decode.cuh").write_text(text + "\nstatic constexpr int kEdit = 1;\n")
    assert bench.captured_traffic("decode_step_kernel", str(path)) is None


def test_committed_summary_names_the_headline_kernel():
    fields = {}
    for line in open(bench.PROFILE_SUMMARY).read().splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    assert fields["kernel"] == "prefill_seq_kernel"
    assert int(fields["traffic_bytes_per_launch"]) > 0
    assert len(fields["source_sha256"]) == 64


def test_profile_cases_cover_the_committed_summaries():
    # every summary under profiles/ names its command; the profile cases it uses exist
    pdir = os.path.join(bench.ROOT, "profiles")
    for name in os.listdir(pdir):
        text = open(os.path.join(pdir, name)).read()
        if "--profile-case" in text:
            used = text.split("--profile-case", 1)[1].split()[0]
            assert used in bench.PROFILE_CASES, (name, used)
