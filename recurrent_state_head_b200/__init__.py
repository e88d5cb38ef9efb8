"""DeltaLog recurrent-state decode on B200 (sm_100a).

The compute path lives in the CUDA library ``libdeltalog.so`` (built from
``csrc/``); ``binding`` is its thin ctypes front end.  Importing the package
loads nothing: the library is opened on first use and a missing or unloadable
library raises at that point.
"""
