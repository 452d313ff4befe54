"""CPU oracle of the MoE block.  Test infrastructure only: imported by the tests, the
smoke check and the CPU-baseline leg of the benchmark, never by the library."""
