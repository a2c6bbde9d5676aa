"""CPU oracle (fp64) for the KroQuant activation quantizer: test
infrastructure, imported only by tests/, __graft_entry__.smoke() and the CPU
legs of bench.py."""
