"""The measured picker table: ``gen_table.py`` turns a sweep record
(``python bench.py --workload sweep`` output, one JSON line per point) into
``csrc/rr_picker_table.h``, which the library compiles in."""
